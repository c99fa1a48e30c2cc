// Angular LSH hash for bf16 inputs on the 5th-generation tensor cores.
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希 and §多輪LSH哈希: for every
// round r, p = x R_r (R_r of size [d, b/2]) and h(x) = argmax([p ; -p]).
//
// Design (persistent, warp-specialised, one CTA per SM):
//   * the rotations of a group of rounds stay resident in shared memory
//     (transposed to K-major by k_hash_prep, loaded once by TMA);
//   * warp 0 streams 128-token tiles of x with TMA (double-buffered);
//   * warp 1 issues tcgen05.mma (M = 128 tokens, N <= 192 columns, K = d)
//     into a ring of TMEM accumulators (two, or four when N <= 128), so the
//     next units' MMAs overlap the epilogue of the current one;
//   * warps 2..13 read the fp32 projections with tcgen05.ld and keep, per
//     token, the largest and second largest |p_j|, the argmax and its sign
//     (three warps per TMEM lane quadrant, each on a contiguous range of at
//     most four 16-column batches, all loaded before one wait). The
//     accumulator is handed back to the MMA as soon as a warp's loads are
//     done, and ||x|| is summed by the warps that do not decide. When a
//     round is one unit of at most 128 columns (b <= 256), the three warps of
//     a quadrant instead take whole units in turn, each deciding its own
//     rounds with no combine (the per-round top-two and combine would
//     otherwise cost more than the round's columns).
// Exactness: the fp32 accumulation of d bf16 products is within
// d * 2^-23 * sum_k |x_k R_kj| <= d * 2^-23 * ||x|| ||R_j|| of the exact sum,
// whatever the order or rounding of the additions. Two columns can only
// trade places when their computed |p| are closer than the sum of their two
// errors, so when the top two |p| are closer than twice that bound
// (kTieFactor; ||x|| and the column norms enter it rounded up) the token is
// queued and k_hash_refine re-decides it in fp64 in the sequential order of
// the definition, so the bucket equals the exact argmax bit for bit.
#pragma once

#include "common.cuh"
#include "hash_exact.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kHashTile = 128;       // tokens per tile (MMA M)
constexpr int kHashEpiPerQuad = 3;   // epilogue warps per TMEM lane quadrant
constexpr int kHashMaxBatches = 4;   // 16-column batches per epilogue warp and unit
constexpr int kHashMaxN = 16 * kHashMaxBatches * kHashEpiPerQuad;  // columns per MMA (N): 192
constexpr int kHashWarps = 2 + 4 * kHashEpiPerQuad;  // 0: TMA, 1: MMA, rest: epilogue
// the norm pass of the attention forms ||x||^2 in this epilogue's order
static_assert(kHashEpiPerQuad - 1 == kNormParts, "norm summation orders must agree");
constexpr float kTieFactor = 2.0f;   // margin threshold / accumulation error bound
constexpr int kHashSmemBudget = 227 * 1024;

struct HashTcPlan {
  int d, kh;        // head dim and its 64-element halves
  int half, nc, ch; // nb/2, MMA N, column chunks per round
  int group;        // rounds resident per CTA
  int groups;       // ceil(rounds / group)
  int tmem_cols;    // per accumulator buffer (power of two >= 32)
  int upw;          // 1: a round is one unit of <= 128 columns, taken whole by one warp
  int stages;       // TMEM accumulators in the MMA -> epilogue ring (2, or 4 when upw)
  size_t smem;      // dynamic shared memory
  size_t x_bytes, r_bytes;
};

// Shared-memory plan; group == 0 when even one round's R does not fit.
inline HashTcPlan hash_tc_plan(int d, int nb, int rounds) {
  HashTcPlan p{};
  p.d = d;
  p.kh = d / 64;
  p.half = nb / 2;
  int nc = ((p.half + 15) / 16) * 16;
  p.nc = nc > kHashMaxN ? kHashMaxN : nc;
  p.ch = (p.half + p.nc - 1) / p.nc;
  p.x_bytes = (size_t)2 * p.kh * kHashTile * 128;
  const size_t per_round = (size_t)p.ch * p.kh * p.nc * 128;
  const size_t misc = 1024 /* alignment */ + 16384 /* barriers, combine buffers */;
  const size_t avail = kHashSmemBudget > (long)(p.x_bytes + misc)
                           ? kHashSmemBudget - p.x_bytes - misc
                           : 0;
  int g = (int)(avail / per_round);
  if (g > rounds) g = rounds;
  p.group = g;
  p.groups = g > 0 ? (rounds + g - 1) / g : 0;
  p.r_bytes = per_round * (size_t)g;
  int tc = 32;
  while (tc < p.nc) tc <<= 1;
  p.tmem_cols = tc;
  p.upw = (p.ch == 1 && p.nc <= 128) ? 1 : 0;
  p.stages = p.upw ? 4 : 2;  // 4 x 128 columns at most: the whole TMEM
  p.smem = p.x_bytes + p.r_bytes + misc;
  return p;
}

// ---------------------------------------------------------------------------
// R [rounds][d][half] -> Rt [rounds][ch * nc][d]: K-major rows for the MMA's
// B operand, each round padded with zero rows to whole chunks of nc. Also,
// per round, an upper bound of max_j ||R_j|| (float bits in rnorm_bits[r],
// zeroed before the launch). A CTA transposes kPrepCols columns through
// shared memory: a warp per column sums its squares in fp64 (rounded up at
// the end, so any summation order gives an upper bound), and each output row
// leaves as 16-byte stores. grid (ceil(ch * nc / kPrepCols), rounds), block
// 256; d <= 128.
constexpr int kPrepCols = 8;
__global__ void __launch_bounds__(256)
    k_hash_prep(const __nv_bfloat16* __restrict__ R, __nv_bfloat16* __restrict__ Rt,
                uint32_t* __restrict__ rnorm_bits, int d, int half, int rows_per_round) {
  __shared__ __align__(16) __nv_bfloat16 tile[kPrepCols][128 + 8];  // [column][k]
  const int r = blockIdx.y;
  const int j0 = blockIdx.x * kPrepCols;
  const __nv_bfloat16* src = R + (int64_t)r * d * half;
  for (int e = threadIdx.x; e < d * kPrepCols; e += blockDim.x) {
    const int k = e / kPrepCols, jj = e % kPrepCols;
    tile[jj][k] = (j0 + jj < half) ? src[(int64_t)k * half + j0 + jj] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < kPrepCols && j0 + warp < half) {
    double ss = 0.0;
    for (int k = lane; k < d; k += 32) {
      const double f = (double)__bfloat162float(tile[warp][k]);
      ss += f * f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) {
      const float nrm = __double2float_ru(sqrt(ss));  // rounded up: an upper bound
      atomicMax(rnorm_bits + r, __float_as_uint(nrm));  // non-negative floats order as uints
    }
  }
  // row jj of the output: d / 8 pieces of 16 bytes
  const int pieces = d / 8;
  __nv_bfloat16* dst = Rt + ((int64_t)r * rows_per_round + j0) * d;
  for (int e = threadIdx.x; e < kPrepCols * pieces; e += blockDim.x) {
    const int jj = e / pieces, c = e % pieces;
    if (j0 + jj < rows_per_round)
      *reinterpret_cast<uint4*>(dst + (int64_t)jj * d + c * 8) =
          *reinterpret_cast<const uint4*>(&tile[jj][c * 8]);
  }
}

// ---------------------------------------------------------------------------
// Exact fp64 re-decision of queued tokens. The queue of round r holds row
// indices bh * n + t at queue + r * cap; its length is count[r]. A CTA takes
// kRefineBatch entries of one round at a time, so each element of the
// transposed rotation is converted to fp64 once per batch. Every thread sums
// whole columns in increasing k, so p_j is the same fp64 number a sequential
// evaluation of the definition gives (bf16 products are exact in fp64).
// grid (ctas per round, rounds), block 128.
constexpr int kRefineBatch = 8;

template <int D>
__global__ void __launch_bounds__(128)
    k_hash_refine(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Rt,
                  const uint64_t* __restrict__ queue, int64_t cap, int32_t* __restrict__ buckets,
                  int n, int nb, int rounds, int rows_per_round, const WsHeader* __restrict__ hdr,
                  int32_t* __restrict__ hist, int sort_tile, int sort_tiles) {
  constexpr int E = kRefineBatch;
  __shared__ double xs[E][D];
  __shared__ double wv[4][E];
  __shared__ int wi[4][E];
  const int r = blockIdx.y;
  const int half = nb / 2;
  const uint32_t count = hdr->pad[16 + r];
  const uint64_t* qr = queue + r * cap;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const __nv_bfloat16* Rr = Rt + (int64_t)r * rows_per_round * D;
  for (uint32_t e0 = blockIdx.x * E; e0 < count; e0 += gridDim.x * E) {
    const int ne = min(E, (int)(count - e0));
    for (int i = tid; i < E * D; i += 128) {
      const int e = i / D, k = i % D;
      xs[e][k] = e < ne ? (double)__bfloat162float(x[(int64_t)qr[e0 + e] * D + k]) : 0.0;
    }
    __syncthreads();
    double bv[E];
    int bi[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      bv[e] = -INFINITY;
      bi[e] = 0x7fffffff;
    }
    // register tile: C columns x E tokens per thread; every column's sum still
    // runs over k = 0..d-1 in order
    constexpr int C = 4;
    for (int j0 = tid; j0 < half; j0 += 128 * C) {
      double acc[C][E];
      const uint4* rr[C];
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const int j = min(j0 + 128 * c, half - 1);
        rr[c] = reinterpret_cast<const uint4*>(Rr + (int64_t)j * D);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[c][e] = 0.0;
      }
      // the next 8 k of every column are loaded while these are summed
      uint4 nxt[C];
#pragma unroll
      for (int c = 0; c < C; ++c) nxt[c] = __ldg(rr[c]);
#pragma unroll 1
      for (int k8 = 0; k8 < D / 8; ++k8) {
        float f[C][8];
#pragma unroll
        for (int c = 0; c < C; ++c) {
          Vec16<__nv_bfloat16>::unpack(nxt[c], f[c]);
          if (k8 + 1 < D / 8) nxt[c] = __ldg(rr[c] + k8 + 1);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          double xv[E];
#pragma unroll
          for (int e = 0; e < E; ++e) xv[e] = xs[e][k8 * 8 + u];
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const double rv = (double)f[c][u];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[c][e] = fma(xv[e], rv, acc[c][e]);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const int j = j0 + 128 * c;
        if (j < half) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            argmax_update(acc[c][e], j, bv[e], bi[e]);
            argmax_update(-acc[c][e], half + j, bv[e], bi[e]);
          }
        }
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv[e], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi[e], o);
        argmax_update(ov, oi, bv[e], bi[e]);
      }
      if (lane == 0) {
        wv[warp][e] = bv[e];
        wi[warp][e] = bi[e];
      }
    }
    __syncthreads();
    if (tid < ne) {
      double v = wv[0][tid];
      int b = wi[0][tid];
      for (int w = 1; w < 4; ++w) argmax_update(wv[w][tid], wi[w][tid], v, b);
      const int64_t row = (int64_t)qr[e0 + tid];
      const int64_t bh = row / n;
      const int t = (int)(row % n);
      int32_t* slot = buckets + (bh * rounds + r) * n + t;
      if (hist != nullptr) {  // move the count of a token whose bucket changed
        const int old = *slot;
        if (old != b) {
          int32_t* hs = hist + (bh * rounds + r) * (int64_t)nb * sort_tiles + t / sort_tile;
          atomicAdd(hs + (int64_t)old * sort_tiles, -1);
          atomicAdd(hs + (int64_t)b * sort_tiles, 1);
        }
      }
      *slot = b;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
struct HashTcArgs {
  int32_t* buckets;   // [BH][rounds][n]
  uint64_t* refine;   // near-tie queues, one of `cap` entries per round
  int64_t cap;        // BH * n
  WsHeader* hdr;      // rnorm bits in hdr->pad[0, 16), queue lengths in hdr->pad[16, 32)
  int32_t* hist;      // the sort's [seg][nb][sort_tiles] counts (zeroed), or null
  float* pinv;        // [BH][n] 1/||x|| by position (the attention's key scales), or null
  int n, nb, rounds, tiles_per_seq, tiles, ctas_per_group;
  int sort_tile, sort_tiles;  // tokens per sort tile, sort tiles per sequence
};

// Running top-2 of |p| with the argmax and its signed value.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Top-two tracker of |p_j| over one token's columns, fed 16 columns at a
// time. Per batch it takes the maxima of the two 8-column halves (trees of
// three-input max operations) and, only when the batch maximum leads, keeps
// the leading half's signed values and the other half's maximum; the argmax,
// its sign and the largest value beside it are found once, in the kept half,
// when the round is done. The second largest |p| overall is the largest of
// that in-half value, the other half's maximum and the largest maximum of the
// other batches, so the result equals a column-by-column top-two scan. Ties
// keep the lower columns (the earlier batch, then the lower half). Columns
// past b/2 (zero rows of the padded rotation) give p = 0 exactly and never
// lead: the first of equal maxima keeps the lead, and a zero maximum is a
// tie that is re-decided.
struct BatchLead {
  float m1;    // largest |p| so far (-1 before the first batch)
  float m2o;   // largest batch maximum outside the lead batch
  float j0;    // first column of the kept half (exact in fp32)
  float o;     // largest |p| of the lead batch's other half
  float s[8];  // the kept half's signed values
  __device__ __forceinline__ void reset() {
    m1 = -1.f;
    m2o = 0.f;
    j0 = 0.f;
    o = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] = 0.f;
  }
  // Batch of 16 values starting at column jb.
  __device__ __forceinline__ void add(const uint32_t (&v)[16], float jb) {
    float w[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) w[k] = __uint_as_float(v[k]);
    const float lo = fmax3(fmax3(fabsf(w[0]), fabsf(w[1]), fabsf(w[2])),
                           fmax3(fabsf(w[3]), fabsf(w[4]), fabsf(w[5])),
                           fmaxf(fabsf(w[6]), fabsf(w[7])));
    const float hi = fmax3(fmax3(fabsf(w[8]), fabsf(w[9]), fabsf(w[10])),
                           fmax3(fabsf(w[11]), fabsf(w[12]), fabsf(w[13])),
                           fmaxf(fabsf(w[14]), fabsf(w[15])));
    const float bm = fmaxf(lo, hi);
    const bool lead = bm > m1;        // the earlier batch keeps the lead on a tie
    m2o = fmaxf(m2o, fminf(bm, m1));  // the batch that does not lead
    m1 = fmaxf(m1, bm);
    if (lead) {
      const bool up = hi > lo;  // the lower half keeps the lead on a tie
      j0 = up ? jb + 8.f : jb;
      o = fminf(lo, hi);
#pragma unroll
      for (int k = 0; k < 8; ++k) s[k] = up ? w[8 + k] : w[k];
    }
  }
  // Largest |p|, second largest, argmax column and its signed value; all
  // zero when no batch was added.
  __device__ __forceinline__ void finish(float& om1, float& om2, int& oidx, float& osv) const {
    float a1 = -1.f, a2 = 0.f, sv = 0.f;
    int k1 = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float a = fabsf(s[k]);
      const bool gt = a > a1;  // lowest column on a tie
      a2 = gt ? fmaxf(a2, a1) : fmaxf(a2, a);
      k1 = gt ? k : k1;
      sv = gt ? s[k] : sv;
      a1 = gt ? a : a1;
    }
    if (m1 < 0.f) {
      om1 = 0.f;
      om2 = 0.f;
      oidx = 0;
      osv = 0.f;
    } else {
      om1 = a1;
      om2 = fmaxf(fmaxf(a2, o), m2o);
      oidx = (int)j0 + k1;
      osv = sv;
    }
  }
};

// Merge rule for the per-warp results of one token: the larger first value
// wins (lower column on a tie); the second value is the largest of the rest.
__device__ __forceinline__ void top2_merge(float& m1, float& m2, int& idx, float& sv, float om1,
                                           float om2, int oidx, float osv) {
  if (om1 > m1 || (om1 == m1 && oidx < idx)) {
    m2 = fmaxf(fmaxf(om2, m2), m1);
    m1 = om1;
    idx = oidx;
    sv = osv;
  } else {
    m2 = fmaxf(fmaxf(om2, m2), om1);
  }
}

// One token's decision for round r: bucket id, the sort's histogram count,
// 1/||x|| (first round), and the near-tie test. sst = ||x||^2 in the order of
// the attention's norm pass; rn = the round's bound of max_j ||R_j||.
template <int D>
__device__ __forceinline__ void hash_decide(const HashTcArgs& a, const HashTcPlan& p, int bh, int t,
                                            int r, float m1, float m2, int idx, float sv, float sst,
                                            float rn) {
  if (a.pinv != nullptr && r == 0)  // once per token, from the first round
    a.pinv[(int64_t)bh * a.n + t] = sst > 0.f ? 1.0f / sqrtf(sst) : 0.f;
  // ||x|| rounded up past the fp32 rounding of its square sum
  const float xnorm = sqrtf(sst) * 1.0001f;
  const float tau = kTieFactor * (float)D * 1.1920929e-7f * xnorm * rn;
  const int bucket = idx + (sv < 0.f ? p.half : 0);
  const int64_t at = ((int64_t)bh * a.rounds + r) * a.n + t;
  a.buckets[at] = bucket;
  if (a.hist != nullptr)  // the sort's tile histogram, counted here
    atomicAdd(a.hist + ((int64_t)(bh * a.rounds + r) * a.nb + bucket) * a.sort_tiles +
                  t / a.sort_tile,
              1);
  if (!(m1 - m2 > tau)) {
    atomicAdd(&a.hdr->hash_refined, 1u);
    const uint32_t k = atomicAdd(&a.hdr->pad[16 + r], 1u);
    a.refine[r * a.cap + k] = (uint64_t)((int64_t)bh * a.n + t);
  }
}

// UPW: the plan's upw, as a template parameter so that each form compiles on
// its own.
template <int D, bool UPW>
__global__ void __launch_bounds__(kHashWarps * 32, 1)
    k_hash_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmr,
              HashTcArgs a, HashTcPlan p) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t XBOX = kHashTile * 128;  // bytes of one 64-column box of x
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* xbuf = base;                   // [2][KH][128 rows][128 B]
  unsigned char* rbuf = base + p.x_bytes;       // [group][ch][KH][nc rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(rbuf + p.r_bytes);
  uint64_t* r_full = bars + 0;
  uint64_t* x_full = bars + 1;     // [2]
  uint64_t* x_empty = bars + 3;    // [2]
  uint64_t* acc_full = bars + 5;   // [stages <= 4]
  uint64_t* acc_empty = bars + 9;  // [stages <= 4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  uint64_t* drain = bars + 15;  // MMA issuer: every issued MMA has completed
  volatile int* drain_fail = reinterpret_cast<volatile int*>(bars + 16);
  constexpr int PO = kHashEpiPerQuad - 1;  // warps of a quadrant that report to h = 0
  constexpr int S = UPW ? 4 : 2;  // p.stages
  float4* comb = reinterpret_cast<float4*>(bars + 18);  // [2][4][PO][32]
  float* ssb = reinterpret_cast<float*>(comb + 2 * 4 * PO * 32);  // [2][4][PO][32]
  float* rn_s = ssb + 2 * 4 * PO * 32;                             // [rounds <= 16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x / a.ctas_per_group;
  const int li = blockIdx.x % a.ctas_per_group;
  const int r0 = g * p.group;
  const int gr = min(p.group, a.rounds - r0);  // rounds in this group

  if (threadIdx.x == 0) {
    mbar_init(r_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(x_full + i, 1);
      // MMA commit + the warps that read x: the norm-summing ones, or every
      // epilogue warp when warps take whole units
      mbar_init(x_empty + i, 1 + 4 * (UPW ? kHashEpiPerQuad : PO));
    }
    for (int i = 0; i < S; ++i) {
      mbar_init(acc_full + i, 1);
      // every epilogue warp, or the one warp per quadrant that takes the unit
      mbar_init(acc_empty + i, UPW ? 4 : 4 * kHashEpiPerQuad);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *drain_fail = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < a.rounds)  // per-round bound of max_j ||R_j|| (k_hash_prep)
    rn_s[threadIdx.x] = reinterpret_cast<const float*>(a.hdr->pad)[threadIdx.x];
  if (warp == 1) tmem_alloc(tmem_slot, S * p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmx);
      prefetch_tensormap(&tmr);
      mbar_expect_tx(r_full, (uint32_t)((size_t)gr * p.ch * KH * p.nc * 128));
      for (int rl = 0; rl < gr; ++rl)
        for (int c = 0; c < p.ch; ++c)
          for (int kh = 0; kh < KH; ++kh) {
            unsigned char* dst = rbuf + ((size_t)(rl * p.ch + c) * KH + kh) * p.nc * 128;
            tma_load_2d(dst, &tmr, r_full, kh * 64, ((r0 + rl) * p.ch + c) * p.nc);
          }
      int it = 0;
      int lastx[2] = {-1, -1};  // last phase issued per x buffer
      for (int tile = li; tile < a.tiles; tile += a.ctas_per_group, ++it) {
        const int xb = it & 1, xk = it >> 1;
        if (xk > 0 && !mbar_wait(x_empty + xb, (xk - 1) & 1)) { fail(); break; }
        if (*abort_flag) break;
        const int bh = tile / a.tiles_per_seq;
        const int row0 = bh * a.n + (tile % a.tiles_per_seq) * kHashTile;
        mbar_expect_tx(x_full + xb, KH * XBOX);
        for (int kh = 0; kh < KH; ++kh)
          tma_load_2d(xbuf + (xb * KH + kh) * XBOX, &tmx, x_full + xb, kh * 64, row0);
        lastx[xb] = xk;
      }
      // No copy may still be writing this CTA's shared memory when it exits:
      // wait (bounded) for the rotations and the last phase of each x buffer.
      if (!mbar_wait(r_full, 0)) *drain_fail = 1;
      for (int b = 0; b < 2; ++b)
        if (lastx[b] >= 0 && !mbar_wait(x_full + b, lastx[b] & 1)) *drain_fail = 1;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors of the first K-step of each operand; K-step kk adds a
      // fixed offset, in 16-byte units, to the start-address field in the low
      // word (shared addresses stay below 256 KB, so the field never carries).
      const uint64_t xd0 = desc_kmajor_sw128(smem_u32(xbuf));
      const uint64_t xd1 = desc_kmajor_sw128(smem_u32(xbuf + KH * XBOX));
      const uint64_t rd0 = desc_kmajor_sw128(smem_u32(rbuf));
      const uint32_t desc_hi = (uint32_t)(xd0 >> 32);  // same for every operand
      const uint32_t r_chunk = (uint32_t)(KH * p.nc * 128) >> 4;
      const uint32_t r_half = (uint32_t)(p.nc * 128) >> 4;  // next 64 columns of K
      // the last chunk of a round stops at the first multiple of 16 columns
      // past b/2
      const uint32_t idesc_full = idesc_bf16_f32(kHashTile, p.nc);
      const uint32_t idesc_last =
          idesc_bf16_f32(kHashTile, min(p.nc, (p.half - (p.ch - 1) * p.nc + 15) & ~15));
      bool ok = mbar_wait(r_full, 0);
      if (!ok) fail();
      int it = 0, u = 0;
      for (int tile = li; ok && tile < a.tiles; tile += a.ctas_per_group, ++it) {
        const int xb = it & 1, xk = it >> 1;
        if (!mbar_wait(x_full + xb, xk & 1)) { fail(); break; }
        tc_fence_after();
        const uint32_t a_lo = (uint32_t)(xb ? xd1 : xd0);
        for (int rl = 0; rl < gr && ok; ++rl) {
          for (int c = 0; c < p.ch; ++c, ++u) {
            const int ab = u % S, uk = u / S;
            if (uk > 0 && !mbar_wait(acc_empty + ab, (uk - 1) & 1)) { fail(); ok = false; break; }
            if (*abort_flag) { ok = false; break; }
            tc_fence_after();
            const uint32_t b_lo = (uint32_t)rd0 + (uint32_t)(rl * p.ch + c) * r_chunk;
            const uint32_t d_tmem = tmem + ab * p.tmem_cols;
            const uint32_t idesc = c == p.ch - 1 ? idesc_last : idesc_full;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int kh = kk >> 2, ks = kk & 3;
              const uint64_t adesc =
                  ((uint64_t)desc_hi << 32) | (a_lo + (uint32_t)((kh * XBOX + ks * 32) >> 4));
              const uint64_t bdesc =
                  ((uint64_t)desc_hi << 32) | (b_lo + kh * r_half + (uint32_t)(ks * 2));
              mma_bf16_ss(d_tmem, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(acc_full + ab);
          }
        }
        mma_commit(x_empty + xb);
      }
      // TMEM is freed below: every MMA issued must have completed first
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) *drain_fail = 1;
    }
  } else if (UPW) {
    // ------------------------------------------- epilogue, whole units per warp
    // Unit u (one round of one tile) goes to warp h = u % 3 of every
    // quadrant, which reduces all of its columns, hands the accumulator back
    // after its last loads and decides. Every epilogue warp waits for each x
    // tile and releases it; a warp with a unit of the tile first sums
    // ||x_row||^2 in the attention's norm-pass order (piece cc into part
    // cc % kNormParts, then 0 + part_0 + part_1 + ...).
    const int e = warp - 2;
    const int q = warp & 3;
    const int h = e >> 2;
    const int row = q * 32 + lane;
    const uint32_t tlane = (uint32_t)(q * 32) << 16;
    const int nbc = (p.half + 15) >> 4;  // 16-column batches of a round
    int it = 0, u = 0;
    bool ok = true;
    for (int tile = li; ok && tile < a.tiles; tile += a.ctas_per_group, ++it) {
      const int xb = it & 1, xk = it >> 1;
      const int bh = tile / a.tiles_per_seq;
      const int t = (tile % a.tiles_per_seq) * kHashTile + row;
      // this tile's units are u .. u + gr - 1; this warp's first is at offset
      const int first = (h - u % kHashEpiPerQuad + kHashEpiPerQuad) % kHashEpiPerQuad;
      if (!mbar_wait(x_full + xb, xk & 1)) {
        fail();
        break;
      }
      float sst = 0.f;
      if (first < gr) {
        float part[kNormParts];
#pragma unroll
        for (int pp = 0; pp < kNormParts; ++pp) part[pp] = 0.f;
#pragma unroll
        for (int cc = 0; cc < KH * 8; ++cc) {
          const unsigned char* line = xbuf + (xb * KH + (cc >> 3)) * XBOX + row * 128;
          const uint4 v = *reinterpret_cast<const uint4*>(line + (((cc & 7) ^ (row & 7)) << 4));
          float f[8];
          Vec16<__nv_bfloat16>::unpack(v, f);
#pragma unroll
          for (int k = 0; k < 8; ++k) part[cc % kNormParts] = fmaf(f[k], f[k], part[cc % kNormParts]);
        }
#pragma unroll
        for (int pp = 0; pp < kNormParts; ++pp) sst += part[pp];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(x_empty + xb);
      for (int rl = first; rl < gr; rl += kHashEpiPerQuad) {
        const int uu = u + rl;
        const int ab = uu % S, uk = uu / S;
        if (*abort_flag || !mbar_wait(acc_full + ab, uk & 1)) {
          fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tbase = tmem + tlane + ab * p.tmem_cols;
        BatchLead st;
        st.reset();
        for (int b0 = 0; b0 < nbc; b0 += kHashMaxBatches) {
          const int K = min(kHashMaxBatches, nbc - b0);
          uint32_t V[kHashMaxBatches][16];
#pragma unroll
          for (int k = 0; k < kHashMaxBatches; ++k)
            if (k < K) tmem_ld16(tbase + (b0 + k) * 16, V[k]);
          tmem_wait_ld_regs(V);
          if (b0 + kHashMaxBatches >= nbc) {  // the unit's last loads: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + ab);
          }
#pragma unroll
          for (int k = 0; k < kHashMaxBatches; ++k)
            if (k < K) st.add(V[k], (float)((b0 + k) * 16));
        }
        float m1, m2, sv;
        int idx;
        st.finish(m1, m2, idx, sv);
        if (t < a.n) hash_decide<D>(a, p, bh, t, r0 + rl, m1, m2, idx, sv, sst, rn_s[r0 + rl]);
      }
      u += gr;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;
    const int q = warp & 3;       // TMEM lane quadrant this warp may access
    const int h = e >> 2;         // rank of this warp in its quadrant
    const int row = q * 32 + lane;
    const uint32_t tlane = (uint32_t)(q * 32) << 16;
    int it = 0, u = 0, rc = 0;
    for (int tile = li; tile < a.tiles; tile += a.ctas_per_group, ++it) {
      const int xb = it & 1, xk = it >> 1;
      const int bh = tile / a.tiles_per_seq;
      const int t = (tile % a.tiles_per_seq) * kHashTile + row;
      // A failure anywhere sets abort_flag; the quadrant's warps OR it at
      // their combine barrier and leave the loop together after it.
      bool ok = true;
      // ||x_row||^2 in parts: warp h >= 1 sums the row's 16-byte chunks
      // cc = h - 1 (mod PO) from the swizzled tile (chunk c of a 128-byte
      // line sits at slot c ^ (row % 8)). Warp h = 0, which decides, reads
      // the partial sums at each round's combine.
      float ss = 0.f;
      if (h > 0) {
        if (!mbar_wait(x_full + xb, xk & 1)) {
          fail();
          ok = false;
        } else {
#pragma unroll 2
          for (int cc = h - 1; cc < KH * 8; cc += PO) {
            const unsigned char* line = xbuf + (xb * KH + (cc >> 3)) * XBOX + row * 128;
            const uint4 v = *reinterpret_cast<const uint4*>(line + (((cc & 7) ^ (row & 7)) << 4));
            float f[8];
            Vec16<__nv_bfloat16>::unpack(v, f);
#pragma unroll
            for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(x_empty + xb);
        }
      }
      bool stop = false;
      for (int rl = 0; rl < gr; ++rl, ++rc) {
        BatchLead st;
        st.reset();
        for (int c = 0; ok && c < p.ch; ++c, ++u) {
          const int ab = u % S, uk = u / S;
          if (!mbar_wait(acc_full + ab, uk & 1)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tbase = tmem + tlane + ab * p.tmem_cols;
          // The chunk's batches are split over the quadrant's warps, at
          // most kHashMaxBatches each, the larger shares to the higher ranks
          // (h = 0 also decides). A warp's loads are issued together and
          // waited for once: one TMEM round trip per unit.
          const int nbc = (min(p.nc, p.half - c * p.nc) + 15) >> 4;
          const int base = nbc / kHashEpiPerQuad, extra_from = kHashEpiPerQuad - nbc % kHashEpiPerQuad;
          const int K = base + (h >= extra_from ? 1 : 0);
          const int b_lo = h * base + max(0, h - extra_from);
          uint32_t V[kHashMaxBatches][16];
#pragma unroll
          for (int k = 0; k < kHashMaxBatches; ++k)
            if (k < K) tmem_ld16(tbase + (b_lo + k) * 16, V[k]);
          tmem_wait_ld_regs(V);
          // the values are in registers: the accumulator is free for the MMA
          // of the unit after next while they are reduced
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + ab);
          const float jb0 = (float)(c * p.nc + b_lo * 16);
#pragma unroll
          for (int k = 0; k < kHashMaxBatches; ++k)
            if (k < K) st.add(V[k], jb0 + 16.f * (float)k);
        }
        float m1, m2, sv;
        int idx;
        st.finish(m1, m2, idx, sv);
        // combine the warps of this quadrant, then decide
        float4* slot = comb + (((rc & 1) * 4 + q) * PO) * 32 + lane;
        float* sslot = ssb + (((rc & 1) * 4 + q) * PO) * 32 + lane;
        if (h > 0) {
          slot[(h - 1) * 32] = make_float4(m1, m2, __int_as_float(idx), sv);
          sslot[(h - 1) * 32] = ss;
        }
        // the quadrant's warps decide together whether to stop (a failure
        // anywhere sets abort_flag), so they leave after the same barrier
        stop = bar_sync_any(1 + q, 32 * kHashEpiPerQuad, *abort_flag != 0);
        if (stop) break;
        if (h == 0) {
#pragma unroll
          for (int o_ = 0; o_ < PO; ++o_) {
            const float4 o = slot[o_ * 32];
            top2_merge(m1, m2, idx, sv, o.x, o.y, __float_as_int(o.z), o.w);
          }
          if (t < a.n) {
            float sst = 0.f;
#pragma unroll
            for (int o_ = 0; o_ < PO; ++o_) sst += sslot[o_ * 32];
            hash_decide<D>(a, p, bh, t, r0 + rl, m1, m2, idx, sv, sst, rn_s[r0 + rl]);
          }
        }
      }
      if (stop) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  // after a drain that gave up, TMEM is left allocated rather than freed
  // under a running MMA; the status word already records the timeout
  if (warp == 1 && !*drain_fail) {
    tc_fence_after();
    tmem_dealloc(tmem, S * p.tmem_cols);
  }
}

}  // namespace lsh
