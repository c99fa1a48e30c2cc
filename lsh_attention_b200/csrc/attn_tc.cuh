// Chunked shared-QK attention on the 5th-generation tensor cores (bf16 in,
// fp32 accumulate), chunk m = 64, reading the rows of x and v by the sort's
// permutation straight from position order: no sorted copies of x and v are
// ever written.
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希注意力 (chunks of m in the
// sorted order), §共享QK中的自掩碼 (self-mask); "Reformer: LSH attention and
// reversible layers" (dtcms.com), §二.1 (unit-length keys, 1/sqrt(d_k)).
// A query in chunk c sees the keys of chunks c-1 and c.
//
// Work unit: a pair of chunks (c0, c0+1) of one (batch, head, round). Its 128
// queries are slots [64 c0, 64 c0 + 128) and its key window is slots
// [64 (c0-1), 64 (c0+2)): the queries are rows 64..191 of the key tile.
// Units of a (batch, head) are numbered round first, then chunk pair; the
// CTAs split every (batch, head)'s units into contiguous runs and walk the
// (batch, head)s in order. So at any time the CTAs work on one (batch,
// head), whose rows all rounds read while they sit in L2 (HBM delivers each
// row about once), and consecutive units of a CTA are consecutive chunk
// pairs of one round: the first 64 rows of a window are the last 64 of the
// previous window, copied inside shared memory instead of gathered again
// (row r + 128 has the swizzle phase of row r), a third fewer rows to fetch.
//
// One persistent CTA per SM, 13 warps:
//   warps 0-1   x loaders: the window's positions (perm) and key norms
//               (1/||x|| by position) are loaded into registers two and one
//               units ahead and written to a 4-deep ring of (logit scale,
//               position) per key; the x rows not carried over go by 16-byte
//               cp.async copies to their places in the 128-byte-swizzled
//               K-major tile (a slot outside [0, n) reads as zero). When a
//               thread's copies have landed it fences them for the async
//               proxy (the tensor cores read shared memory through it) and
//               arrives.
//   warps 2-3   v loaders: the same for the v rows, at the positions of the
//               ring, into the tile of the P.V product.
//   warp 4      tcgen05.mma: S(u+1) = Q K^T into TMEM S[s], then O(u) = P V
//               with P read from TMEM, so S of the next unit is ready when
//               the softmax warps finish the current one. The x tile is free
//               again as soon as S is computed (the ring keeps the metadata).
//   warps 5-8   softmax, one query row per thread, one pass: logits in log2
//               units are bounded by ||q|| log2(e) / sqrt(d) (keys have unit
//               length), which serves as the stabiliser, so every probability
//               is exp2(l - bound) <= 1 and is written to TMEM (bf16, over the
//               dead S columns) as soon as it is computed; the row sum goes to
//               the epilogue. A row whose only visible key is itself (the -1e5
//               self logit) is flagged: its output is v of the query itself.
//   warps 9-12  epilogue: O from TMEM, divided by the row sum and packed to
//               bf16 (the accumulator is released before the stores), staged
//               per warp in a 4 KB swizzled buffer (32 rows x 64 columns) and
//               written by TMA bulk stores (slot order); the softmax writes lse
//               at the query's position. Each round's output is kept in bf16:
//               its rounding (relative 2^-9, before a convex combination over
//               the rounds) is of the size of the final bf16 rounding of out.
// TMEM: S[0] = [0, 192), S[1] = [192, 384), O = [384, 384 + d).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kAttnM = 64;      // chunk length served by this kernel
constexpr int kAttnKeys = 192;  // key window of a pair of chunks
constexpr int kAttnWarps = 13;
constexpr int kAttnStats = 4;   // row-sum slots between softmax and epilogue
constexpr int kAttnRing = 4;    // metadata ring depth
// Above this bound (log2 units) the stabiliser could push exp2 below the
// normal range: those rows use their exact maximum instead.
constexpr float kAttnBoundMax = 60.f;

struct AttnTcArgs {
  const __nv_bfloat16* x;      // [BH][n][d] position order
  const __nv_bfloat16* v;      // [BH][n][d] position order
  const float* pinv;           // [BH][n] 1/||x|| by position (0 for a zero row)
  const int32_t* perm;         // [S][n] position of each slot
  float* lse;                  // [S][n] each round's lse by position (the caller's output)
  WsHeader* hdr;
  int n, rounds, pairs_per_seg;
  int units;                   // BH * pairs_per_seg * rounds
};

// One unit of work: a pair of chunks (first chunk c0) of segment seg =
// (batch-head bh, round).
struct AttnUnit {
  int bh, seg, c0;
};

// 2^x by the hardware's approximate base-2 exponential (relative error near
// 2^-22, results below 2^-126 flushed to zero). The arguments here are <= 0
// (logit minus an upper bound) and the results are rounded to bf16.
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kAttnWarps * 32, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmo, AttnTcArgs a) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t BOX = kAttnKeys * 128;
  constexpr uint32_t TILE = KH * BOX;
  constexpr int ROWS = kAttnKeys / 64;  // window rows per x-loader thread (metadata)
  constexpr int CPR = KH * 8;            // 16-byte pieces per row
  constexpr int RSTEP = 64 / CPR;        // rows between a loader thread's pieces
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int kNoKey = 0x7fffffff;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // tiles of x and of v in flight: three at d = 64 (small tiles), so a unit's
  // rows can be gathered while the two before it are still in use
  constexpr int NB = D == 64 ? 3 : 2;
  unsigned char* xt = base;                                           // [NB][KH][192][128 B]
  unsigned char* vt = base + NB * TILE;                               // [NB][KH][192][128 B]
  unsigned char* ostage = base + 2 * NB * TILE;                       // [4 warps][32][128 B]
  float2* ktab = reinterpret_cast<float2*>(ostage + 4 * 32 * 128);    // [ring][192] (scale, pos)
  float* rstat = reinterpret_cast<float*>(ktab + kAttnRing * kAttnKeys);  // [4][128] 1/sum
  uint64_t* bars = reinterpret_cast<uint64_t*>(rstat + kAttnStats * 128);
  uint64_t* xfull = bars + 36;   // [NB] x rows landed (64 x-loader threads)
  uint64_t* xfree = bars + 39;   // [NB] S MMA done with the x tile
  uint64_t* vfull = bars + 42;   // [NB] v rows landed (64 v-loader threads)
  uint64_t* vfree = bars + 45;   // [NB] PV MMA done with the v tile
  uint64_t* sfull = bars + 8;    // [2] S MMA done
  uint64_t* pready = bars + 10;  // [2] P written (4 softmax warps)
  uint64_t* sfree = bars + 12;   // [2] PV MMA done with P
  uint64_t* ofull = bars + 14;   // PV MMA done
  uint64_t* ofree = bars + 15;   // 4 epilogue warps done reading O
  uint64_t* statf = bars + 16;   // [4] row sums written (4 softmax warps)
  uint64_t* mfull = bars + 20;   // [ring] metadata written (64 x-loader threads)
  uint64_t* mfree = bars + 24;   // [ring] 4 softmax warps and 2 v-loader warps done with it
  uint64_t* drain = bars + 28;   // MMA issuer: every issued MMA has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 29);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 30);
  volatile int* drain_fail = reinterpret_cast<volatile int*>(bars + 31);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's units: for every (batch, head) the run [lo, lo + cnt) of its P
  // units; when P < G (short sequences) one run of the whole list instead.
  // Unit, slot and segment numbers fit in 32 bits (segments x n < 2^31).
  const int P = a.rounds * a.pairs_per_seg, G = gridDim.x;
  const bool per_head = P >= G;
  const int lo = (int)(per_head ? (int64_t)blockIdx.x * P / G : (int64_t)blockIdx.x * a.units / G);
  const int cnt = (int)(per_head ? (int64_t)(blockIdx.x + 1) * P / G - lo
                                 : (int64_t)(blockIdx.x + 1) * a.units / G - lo);
  const int nu = per_head ? (a.units / P) * cnt : cnt;
  if (nu == 0) return;  // uniform across the CTA

  if (tid == 0) {
    for (int i = 0; i < NB; ++i) {
      mbar_init(xfull + i, 64);
      mbar_init(xfree + i, 1);
      mbar_init(vfull + i, 64);
      mbar_init(vfree + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sfull + i, 1);
      mbar_init(pready + i, 4);
      mbar_init(sfree + i, 1);
    }
    mbar_init(ofull, 1);
    mbar_init(ofree, 4);
    for (int i = 0; i < kAttnStats; ++i) mbar_init(statf + i, 4);
    for (int i = 0; i < kAttnRing; ++i) {
      mbar_init(mfull + i, 64);
      mbar_init(mfree + i, 4 + 2);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *drain_fail = 0;
    fence_mbar_init();
  }
  if (warp == 4) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem + 384;
  const float c_scale = kLog2e / sqrtf((float)D);

  auto fail = [&]() {
    record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
    *abort_flag = 1;
  };
  // this CTA's unit i (32-bit unsigned divisions)
  auto unit_of = [&](int i) {
    AttnUnit u;
    int q;
    if (per_head) {
      u.bh = (int)((unsigned)i / (unsigned)cnt);
      q = lo + i - u.bh * cnt;
    } else {
      const int g = lo + i;
      u.bh = (int)((unsigned)g / (unsigned)P);
      q = g - u.bh * P;
    }
    const int r = (int)((unsigned)q / (unsigned)a.pairs_per_seg);
    u.seg = u.bh * a.rounds + r;
    u.c0 = 2 * (q - r * a.pairs_per_seg);
    return u;
  };

  if (warp < 4) {
    // ------------------------------------------------------------ loaders
    const bool xl = warp < 2;      // x loaders also write the ring
    const int lt = tid & 63;       // rank among this loader pair of warps
    const unsigned char* src0 = reinterpret_cast<const unsigned char*>(xl ? a.x : a.v);
    unsigned char* tiles = xl ? xt : vt;
    uint64_t* full = xl ? xfull : vfull;
    uint64_t* tfree = xl ? xfree : vfree;
    const int piece = lt % CPR;    // this thread's 16-byte piece of every row it copies
    const int kh = piece >> 3, cc = piece & 7;
    // x loaders: positions (perm) of the window rows lt + 64 t of a unit and
    // their logit scales (1/||x|| c); the loads are issued two units (perm)
    // and one unit (norms) before the values go to the ring. Every load reads
    // a valid address and its value is first used a unit later (validity
    // comes from the slot number, which needs no load), so the loop never
    // waits for one.
    auto perm_of = [&](bool live, const AttnUnit& u, int (&raw)[ROWS], uint32_t& ok) {
      ok = 0u;
#pragma unroll
      for (int t = 0; t < ROWS; ++t) {
        const int ks = live ? (u.c0 - 1) * kAttnM + lt + 64 * t : -1;
        const bool in = ks >= 0 && ks < a.n;
        ok |= (in ? 1u : 0u) << t;
        raw[t] = __ldg(a.perm + (int64_t)u.seg * a.n + (in ? ks : 0));
      }
    };
    auto checked = [&](const int (&raw)[ROWS], uint32_t ok, int (&p)[ROWS]) {
#pragma unroll
      for (int t = 0; t < ROWS; ++t) p[t] = (ok >> t) & 1u ? raw[t] : kNoKey;
    };
    auto norm_of = [&](const AttnUnit& u, const int (&p)[ROWS], float (&raw)[ROWS]) {
#pragma unroll
      for (int t = 0; t < ROWS; ++t)
        raw[t] = __ldg(a.pinv + (int64_t)u.bh * a.n + (p[t] != kNoKey ? p[t] : 0));
    };
    // Gather N window rows (first, first + RSTEP, ...) of this thread's piece:
    // every position is read from the ring first, then the copies are issued
    // back to back.
    auto gather = [&](auto n_rows, int first, const float2* kt, unsigned char* dk,
                      const unsigned char* rows) {
      constexpr int N = decltype(n_rows)::value;
      constexpr int B = N < 8 ? N : 8;  // rows per batch (keeps the code small)
#pragma unroll 1
      for (int g = 0; g < N; g += B) {
        int pos[B];
#pragma unroll
        for (int k = 0; k < B; ++k) pos[k] = __float_as_int(kt[first + (g + k) * RSTEP].y);
#pragma unroll
        for (int k = 0; k < B; ++k) {
          const int row = first + (g + k) * RSTEP;
          const bool valid = pos[k] != kNoKey;
          cp_async16_zfill(dk + row * 128 + ((cc ^ (row & 7)) << 4),
                           valid ? rows + (int64_t)pos[k] * (D * 2) : src0, valid);
        }
      }
    };
    // units i - 1 .. i + 3
    AttnUnit u_prev = unit_of(0), u_cur = u_prev, u_n1 = unit_of(1), u_n2 = unit_of(2),
             u_n3 = unit_of(3);
    // p0, p1: positions of units i, i + 1; r2: raw positions of unit i + 2;
    // n0, n1: raw norms of units i, i + 1
    int p0[ROWS], p1[ROWS], r2[ROWS];
    float n0[ROWS], n1[ROWS];
    uint32_t ok2 = 0u;
    if (xl) {
      perm_of(true, u_cur, r2, ok2);
      checked(r2, ok2, p0);
      perm_of(1 < nu, u_n1, r2, ok2);
      checked(r2, ok2, p1);
      norm_of(u_cur, p0, n0);
      norm_of(u_n1, p1, n1);
      perm_of(2 < nu, u_n2, r2, ok2);
    }
    // Unit i's copies are issued before unit i - 1's are awaited, so two
    // tiles' gathers are in flight per loader thread; unit i - 1's tile is
    // handed to the tensor cores (and its last 64 rows carried into unit i's
    // tile) once they have landed.
    const int pair_bar = 2 + (xl ? 0 : 1);
    bool stopped = false;
    for (int i = 0; i < nu; ++i) {
      const int s = i % NB, k = i / NB, m = i & (kAttnRing - 1), km = i / kAttnRing;
      const int sp = (i + NB - 1) % NB;  // tile of unit i - 1
      bool got;
      if (xl)  // ring slot m free (unit i - 4 done with it), x tile s free (S of unit i - NB)
        got = (km == 0 || mbar_wait(mfree + m, (km - 1) & 1)) &&
              (k == 0 || mbar_wait(tfree + s, (k - 1) & 1));
      else     // ring slot m written for unit i, v tile s free (PV of unit i - NB)
        got = mbar_wait(mfull + m, km & 1) && (k == 0 || mbar_wait(tfree + s, (k - 1) & 1));
      if (!got) fail();
      // both warps of the pair stop together (a failure anywhere sets abort_flag)
      if (bar_sync_any(pair_bar, 64, !got || *abort_flag)) {
        stopped = true;
        break;
      }
      float2* kt = ktab + m * kAttnKeys;
      if (xl) {
#pragma unroll
        for (int t = 0; t < ROWS; ++t)
          kt[lt + 64 * t] =
              make_float2(p0[t] != kNoKey ? n0[t] * c_scale : 0.f, __int_as_float(p0[t]));
        bar_sync_any(2, 64, false);  // the pair's ring entries are written
        mbar_arrive(mfull + m);
      }
      unsigned char* dst = tiles + s * TILE;
      // rows 0..63 = rows 128..191 of the previous tile
      const bool carry = i > 0 && u_cur.seg == u_prev.seg && u_cur.c0 == u_prev.c0 + 2;
      const unsigned char* rows = src0 + (int64_t)u_cur.bh * a.n * (D * 2) + piece * 16;
      unsigned char* dk = dst + kh * BOX;
      if (!carry) gather(std::integral_constant<int, kAttnM / RSTEP>{}, lt / CPR, kt, dk, rows);
      gather(std::integral_constant<int, (kAttnKeys - kAttnM) / RSTEP>{}, kAttnM + lt / CPR, kt,
             dk, rows);
      cp_async_commit();
      if (!xl) {  // done reading the ring slot
        __syncwarp();
        if (lane == 0) mbar_arrive(mfree + m);
      } else {  // the next units' metadata: norms one unit ahead, positions two
#pragma unroll
        for (int t = 0; t < ROWS; ++t) {
          p0[t] = p1[t];
          n0[t] = n1[t];
        }
        checked(r2, ok2, p1);   // unit i + 2's positions, loaded a unit ago
        norm_of(u_n2, p1, n1);
        perm_of(i + 3 < nu, u_n3, r2, ok2);
      }
      if (i > 0) {
        cp_async_wait_prev();  // this thread's copies of unit i - 1 have landed
        if (carry) {
          bar_sync_any(pair_bar, 64, false);  // ... and the whole pair's
          const unsigned char* prev = tiles + sp * TILE;
          // every piece is loaded before the first is stored (8 at a time)
          constexpr int NP = kAttnM * 8 * KH / 64;  // pieces per thread
#pragma unroll
          for (int g = 0; g < NP; g += 8) {
            uint4 buf[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int e = lt + 64 * (g + j);
              const int h = e / (kAttnM * 8), rc = e % (kAttnM * 8);  // piece rc of half h
              buf[j] = *reinterpret_cast<const uint4*>(prev + h * BOX + 128 * 128 + rc * 16);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int e = lt + 64 * (g + j);
              const int h = e / (kAttnM * 8), rc = e % (kAttnM * 8);
              *reinterpret_cast<uint4*>(dst + h * BOX + rc * 16) = buf[j];
            }
          }
        }
        fence_proxy_async_smem();  // unit i - 1's rows (and unit i's carried ones) for the MMA
        mbar_arrive(full + sp);
      }
      u_prev = u_cur;
      u_cur = u_n1;
      u_n1 = u_n2;
      u_n2 = u_n3;
      u_n3 = unit_of(i + 4);
    }
    cp_async_wait_all();  // nothing of this thread's still writes shared memory at exit
    if (!stopped) {  // the last unit
      fence_proxy_async_smem();
      mbar_arrive(full + ((nu - 1) % NB));
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kAttnKeys);
      const uint32_t idesc_o = idesc_bf16_f32(128, D) | (1u << 16);  // B = V, MN-major
      auto issue_s = [&](int i) {
        const int s = i & 1, k = i >> 1;     // S in TMEM
        const int tb = i % NB, tk = i / NB;  // x tile
        if (!mbar_wait(xfull + tb, tk & 1)) return false;
        if (k > 0 && !mbar_wait(sfree + s, (k - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t xa = smem_u32(xt + tb * TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kh = kk >> 2, ks = kk & 3;
          const uint64_t ad = desc_kmajor_sw128(xa + kh * BOX + kAttnM * 128 + ks * 32);
          const uint64_t bd = desc_kmajor_sw128(xa + kh * BOX + ks * 32);
          mma_bf16_ss(tmem + s * 192, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(sfull + s);
        mma_commit(xfree + tb);
        return true;
      };
      auto issue_pv = [&](int i) {
        const int s = i & 1, k = i >> 1;     // P in TMEM
        const int tb = i % NB, tk = i / NB;  // v tile
        if (!mbar_wait(pready + s, k & 1)) return false;
        if (!mbar_wait(vfull + tb, tk & 1)) return false;
        if (i > 0 && !mbar_wait(ofree, (i - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(vt + tb * TILE);
#pragma unroll
        for (int kk = 0; kk < kAttnKeys / 16; ++kk) {
          const uint64_t bd = desc_mnmajor_sw128(va + kk * 16 * 128, BOX);
          mma_bf16_ts(tm_o, tmem + s * 192 + kk * 8, bd, idesc_o, kk > 0 ? 1u : 0u);
        }
        mma_commit(ofull);
        mma_commit(vfree + tb);
        mma_commit(sfree + s);
        return true;
      };
      bool ok = issue_s(0);
      for (int i = 0; ok && i < nu && !*abort_flag; ++i)
        ok = (i + 1 >= nu || issue_s(i + 1)) && issue_pv(i);
      if (!ok) fail();
      // TMEM is freed below: every MMA issued must have completed first
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) *drain_fail = 1;
    }
  } else if (warp < 9) {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;       // TMEM lane quadrant
    const int row = q * 32 + lane;
    const int wcol = q < 2 ? 0 : kAttnM;  // first in-window key column
    const uint32_t tl = (uint32_t)(q * 32) << 16;
    for (int i = 0; i < nu; ++i) {
      const int s = i & 1, k = i >> 1, m = i & (kAttnRing - 1), km = i / kAttnRing;
      const bool got = mbar_wait(sfull + s, k & 1) && mbar_wait(mfull + m, km & 1);
      if (!got) fail();
      tc_fence_after();
      // the four softmax warps; a failure seen by any of them stops all four
      // here, so none is left waiting at this barrier
      if (bar_sync_any(1, 128, !got || *abort_flag)) break;
      const AttnUnit u = unit_of(i);
      const int64_t seg = u.seg;
      const int c0 = u.c0;
      const float2* kt = ktab + m * kAttnKeys;
      const float2 me = kt[kAttnM + row];
      const int qpos = __float_as_int(me.y);
      // stabiliser: ||q|| log2(e) / sqrt(d) bounds every logit of the row
      float bound = me.x > 0.f ? c_scale * c_scale / me.x : 0.f;
      const uint32_t ts = tmem + tl + s * 192;
      auto visible = [&](int pj) {
        if (CAUSAL) return pj < qpos;            // earlier positions only (not self)
        return pj != qpos && pj != kNoKey;       // every valid key but self
      };
      if (__any_sync(0xffffffffu, bound > kAttnBoundMax)) {
        // rare: exact row maximum as the stabiliser for those rows
        float mx = -INFINITY;
#pragma unroll 1
        for (int b = 0; b < 4; ++b) {
          uint32_t v[32];
          tmem_ld32(ts + wcol + b * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float2 t = kt[wcol + b * 32 + c];
            if (visible(__float_as_int(t.y))) mx = fmaxf(mx, __uint_as_float(v[c]) * t.x);
          }
        }
        if (bound > kAttnBoundMax) bound = mx == -INFINITY ? 0.f : mx;
      }
      float sum0 = 0.f, sum1 = 0.f;
      // 32-key batches per TMEM wait: two at d = 64, where the softmax paces
      // the pipeline (more exponents in flight), one at d = 128
      constexpr int BPW = D == 64 ? 2 : 1;
#pragma unroll 1
      for (int b2 = 0; b2 < 4; b2 += BPW) {
        uint32_t v[BPW][32];
#pragma unroll
        for (int h = 0; h < BPW; ++h) tmem_ld32(ts + wcol + (b2 + h) * 32, v[h]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < BPW; ++h) {
          const int b = b2 + h;
          uint32_t pk[16];
          const float4* kt4 = reinterpret_cast<const float4*>(kt + wcol + b * 32);
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float4 t = kt4[c >> 1];  // (scale, position) of keys c and c + 1
            // every exponent is computed, then invisible keys are masked: no
            // divergent branch per key
            const float e0 = ex2_approx(fmaf(__uint_as_float(v[h][c]), t.x, -bound));
            const float e1 = ex2_approx(fmaf(__uint_as_float(v[h][c + 1]), t.z, -bound));
            const float p0 = visible(__float_as_int(t.y)) ? e0 : 0.f;
            const float p1 = visible(__float_as_int(t.w)) ? e1 : 0.f;
            sum0 += p0;
            sum1 += p1;
            pk[c >> 1] = pack_bf16x2(p0, p1);
          }
          // P column c holds keys 2c, 2c+1: batch b lands in columns
          // [wcol/2 + 16b, wcol/2 + 16b + 16), S columns already read (or,
          // for wcol = 64 and b < 2, columns outside this row's window)
          tmem_st16(ts + wcol / 2 + b * 16, pk);
        }
      }
      uint32_t z[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) z[c] = 0u;
      tmem_st16(ts + (q < 2 ? 64 : 0), z);  // P outside this row's window
      tmem_st16(ts + (q < 2 ? 80 : 16), z);
      tmem_wait_st();
      const float sum = sum0 + sum1;
      const int qs = c0 * kAttnM + row;
      // lse over the visible keys and the self logit; exp(-1e5) vanishes
      // unless the row sees nothing else
      if (qs < a.n)
        a.lse[seg * a.n + qpos] = sum > 0.f ? (bound + log2f(sum)) * 0.6931471805599453f
                                            : kSelfLogit;
      rstat[(i % kAttnStats) * 128 + row] = sum > 0.f ? 1.0f / sum : -1.f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(pready + s);
        mbar_arrive(statf + (i % kAttnStats));
        mbar_arrive(mfree + m);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tl = (uint32_t)(q * 32) << 16;
    for (int i = 0; i < nu; ++i) {
      if (!mbar_wait(ofull, i & 1) || !mbar_wait(statf + (i % kAttnStats), (i / kAttnStats) & 1)) {
        fail();
        break;
      }
      tc_fence_after();
      const float inv = rstat[(i % kAttnStats) * 128 + row];
      // O / sum, packed to bf16 pairs as it leaves TMEM: pk[j] = columns 2j, 2j+1
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
      const AttnUnit u = unit_of(i);
      const int64_t bh = u.bh, seg = u.seg;
      const int c0 = u.c0;
      const int qs0 = c0 * kAttnM + q * 32;  // first query slot of this warp
      if (qs0 < a.n) {  // n % 64 == 0: a warp's 32 rows are all valid or all not
        const uint4* vr = nullptr;
        if (inv <= 0.f)  // only the token itself is visible: its own value row
          vr = reinterpret_cast<const uint4*>(
              a.v + (bh * a.n + a.perm[seg * a.n + qs0 + lane]) * (int64_t)D);
        unsigned char* stg = ostage + (warp - 9) * 32 * 128;
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {  // 64 columns (128 bytes of bf16) per store
          if (lane == 0) bulk_wait_read_all();  // the previous store has read the buffer
          __syncwarp();
          // row `lane`, 16-byte chunk c (columns 64 b + 8 c ...) goes to slot
          // c ^ (lane % 8) (128-byte swizzle)
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
          if (lane == 0) {
            tma_store_2d(&tmo, stg, b * 64, (int)(seg * a.n) + qs0);
            bulk_commit();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  // after a drain that gave up, TMEM is left allocated rather than freed
  // under a running MMA; the status word already records the timeout
  if (warp == 4 && !*drain_fail) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

inline size_t attn_tc_smem(int D) {
  const size_t tile = (size_t)(D / 64) * kAttnKeys * 128;
  const int nb = D == 64 ? 3 : 2;  // NB of the kernel
  return 1024 + 2 * nb * tile + 4 * 32 * 128 + (size_t)kAttnRing * kAttnKeys * 8 +
         kAttnStats * 128 * 4 + 512;
}

// 1/||x|| of every row of x [rows][D] (bf16), for the attention's key scales
// when the hash did not produce them. The square sum is formed in the order
// the tensor-core hash's epilogue forms it (partial sums over the row's
// 16-byte pieces p = r, r + P, r + 2P, ... for r < P = kNormParts, each
// piece's elements in order, then 0 + part_0 + part_1 + ...), so both
// sources give the same bits: a forward gets the same output whether the
// hash runs inside it or the caller passes its bucket ids. A group of
// kNormParts lanes per row.
template <int D>
__global__ void __launch_bounds__(256)
    k_row_invnorm(const __nv_bfloat16* __restrict__ x, float* __restrict__ pinv, int64_t rows) {
  constexpr int L = kNormParts;
  constexpr int PIECES = D / 8;
  const int gl = threadIdx.x % L;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x / L);
  const int64_t warp_first = ((int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) / L;
  for (int64_t r0 = warp_first; r0 < rows; r0 += stride) {
    const int64_t r = r0 + (threadIdx.x & 31) / L;
    float ss = 0.f;
    if (r < rows) {
      const uint4* row = reinterpret_cast<const uint4*>(x + r * D);
      uint4 u[PIECES / L];
#pragma unroll
      for (int k = 0; k < PIECES / L; ++k) u[k] = row[gl + k * L];
#pragma unroll
      for (int k = 0; k < PIECES / L; ++k) {
        float f[8];
        Vec16<__nv_bfloat16>::unpack(u[k], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    // 0 + part_0 + part_1 + ..., in that order
    float sst = 0.f;
#pragma unroll
    for (int o = 0; o < L; ++o) sst += __shfl_sync(0xffffffffu, ss, (threadIdx.x & 31) - gl + o);
    if (r < rows && gl == 0) pinv[r] = sst > 0.f ? 1.0f / sqrtf(sst) : 0.f;
  }
}

}  // namespace lsh
