// Host side of the C ABI declared in include/lsh_attn.h: argument checks,
// workspace carving, and kernel launches on the caller's stream.
#include "lsh_attn.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <stdint.h>
#include <string.h>

#include "attn_dense.cuh"
#include "bwd.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "gather.cuh"
#include "hash_exact.cuh"
#include "hash_tc.cuh"
#include "merge.cuh"
#include "sort.cuh"
#include "tma_host.cuh"
#include "topk.cuh"

namespace {

using namespace lsh;

struct Layout {
  size_t header, buckets, perm, inv, invnorm, pinv, lse_s, hist, xs, vs, out_s, rt, refine,
      total;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Dims {
  int B, H, n, d, nb, m, rounds, causal, dtype;
  int64_t BH, S;  // (batch, head) pairs; segments = BH * rounds
  int esize;
  int tiles;
  bool attention;  // the call runs the chunked attention (the forward)
};

// bf16, chunk 64: the tcgen05 kernel, which reads x and v rows by perm.
inline bool attn_tc_supported(const Dims& D) {
  return D.dtype == LSH_BF16 && D.m == kAttnM && D.n % kAttnM == 0 &&
         D.S * (int64_t)D.n < (int64_t(1) << 31);
}

// `attention`: the call runs the chunked attention, so the chunk length must
// be in the supported set; hash and sort ignore it beyond chunk >= 1.
lsh_status check_desc(const lsh_attn_desc* desc, Dims* D, bool attention) {
  if (!desc) return LSH_ERR_INVALID_ARG;
  const lsh_attn_desc& q = *desc;
  if (q.batch < 1 || q.heads < 1 || q.n < 1 || q.d < 1 || q.n_buckets < 1 || q.chunk < 1 ||
      q.rounds < 1 || (q.causal != 0 && q.causal != 1) || (q.dtype != LSH_F32 && q.dtype != LSH_BF16))
    return LSH_ERR_INVALID_ARG;
  if (q.d != 64 && q.d != 128) return LSH_ERR_UNSUPPORTED;
  if (q.n_buckets % 2 != 0 || q.n_buckets < 2 || q.n_buckets > 4096) return LSH_ERR_UNSUPPORTED;
  if (q.rounds > 16) return LSH_ERR_UNSUPPORTED;
  const int m = q.chunk < q.n ? q.chunk : q.n;
  if (attention && (m > 128 || q.n % m != 0)) return LSH_ERR_UNSUPPORTED;
  if ((int64_t)q.n * q.n_buckets >= (int64_t(1) << 31)) return LSH_ERR_UNSUPPORTED;
  D->B = q.batch;
  D->H = q.heads;
  D->n = q.n;
  D->d = q.d;
  D->nb = q.n_buckets;
  D->m = m;
  D->rounds = q.rounds;
  D->causal = q.causal;
  D->dtype = q.dtype;
  D->BH = (int64_t)q.batch * q.heads;
  D->S = D->BH * q.rounds;
  D->esize = q.dtype == LSH_BF16 ? 2 : 4;
  D->attention = attention;
  const int tile = sort_tile(q.n_buckets);
  D->tiles = (q.n + tile - 1) / tile;
  if (D->S * (int64_t)q.n * q.d >= (int64_t(1) << 40)) return LSH_ERR_UNSUPPORTED;
  if (D->S > 65535) return LSH_ERR_UNSUPPORTED;  // segments index grid.y
  return LSH_OK;
}

Layout layout_of(const Dims& D) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t sn = (size_t)D.S * D.n;
  // the forward's attention reads x and v by perm on the tensor-core path
  // (key scales by position: pinv) and sorted copies otherwise (xs, vs, and
  // key scales by slot: invnorm); hash and sort calls need neither
  const bool tc = D.attention && attn_tc_supported(D);
  const bool copies = D.attention && !tc;
  L.header = take(sizeof(WsHeader));
  L.buckets = take(sn * 4);
  L.perm = take(sn * 4);
  L.inv = take(sn * 4);
  L.invnorm = take(tc ? 0 : sn * 4);  // also written by lsh_attn_sort's row gather
  L.pinv = take(tc ? (size_t)D.BH * D.n * 4 : 0);
  L.lse_s = take(sn * 4);
  L.hist = take((size_t)D.S * D.nb * D.tiles * 4);
  L.xs = take(copies ? sn * D.d * D.esize : 0);
  L.vs = take(copies ? sn * D.d * D.esize : 0);
  L.out_s = take(D.attention ? sn * D.d * D.esize : 0);  // each round's output, input type
  const HashTcPlan hp = hash_tc_plan(D.d, D.nb, D.rounds);
  L.rt = take((size_t)D.rounds * hp.ch * hp.nc * D.d * 2);  // R transposed (bf16 hash)
  L.refine = take(sn * 8);                             // near-tie queue of the bf16 hash
  L.total = off;
  return L;
}

lsh_status check_ws(const Dims& D, const void* ws, size_t ws_bytes, Layout* L) {
  *L = layout_of(D);
  if (!ws || ((uintptr_t)ws & 255) != 0 || ws_bytes < L->total) return LSH_ERR_WORKSPACE;
  return LSH_OK;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

inline lsh_status last_cuda() {
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

lsh_status reset_header(void* ws, cudaStream_t st) {
  return cudaMemsetAsync(ws, 0, sizeof(WsHeader), st) == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

// One CTA waits on an mbarrier that nothing arrives at, with a short limit:
// the wait gives up, the status word records the timeout, the kernel returns.
__global__ void k_wait_selftest(WsHeader* hdr, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sm100::mbar_wait(&bar, 0, limit_ns))
    record_status(hdr, 5u /* LSH_ERR_TIMEOUT */);
}

// ---------------------------------------------------------------- launches
// Profiling marks: the events of lsh_attn_forward_profiled, one per kernel
// boundary (indices in lsh_attn.h).
inline lsh_status mark(void* const* events, int i, cudaStream_t st) {
  if (!events) return LSH_OK;
  return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st) == cudaSuccess ? LSH_OK
                                                                              : LSH_ERR_CUDA;
}

lsh_status launch_hash_exact(const Dims& D, const void* x, const void* R, int32_t* buckets,
                             cudaStream_t st, bool bf16) {
  const int esz = bf16 ? 2 : 4;
  const int xstride = D.d + (esz == 4 ? 1 : 2);
  const size_t smem =
      sizeof(double) * D.d * kHashExactCols + (size_t)esz * kHashExactTokens * xstride;
  dim3 grid((D.n + kHashExactTokens - 1) / kHashExactTokens, (unsigned)D.BH, D.rounds);
  if (bf16) {
    auto kern = k_hash_exact<__nv_bfloat16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return LSH_ERR_CUDA;
    kern<<<grid, kHashExactTokens, smem, st>>>(static_cast<const __nv_bfloat16*>(x),
                                                static_cast<const __nv_bfloat16*>(R), buckets,
                                                D.n, D.d, D.nb, D.rounds);
  } else {
    auto kern = k_hash_exact<float>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return LSH_ERR_CUDA;
    kern<<<grid, kHashExactTokens, smem, st>>>(static_cast<const float*>(x),
                                                static_cast<const float*>(R), buckets, D.n, D.d,
                                                D.nb, D.rounds);
  }
  return last_cuda();
}

// bf16: tcgen05 projection + top-2 screen, fp64 re-decision of near ties.
// hist: when not null, the sort's tile histograms are counted by the hash
// (and *hist_done set); otherwise the sort counts them itself. pinv: when not
// null, 1/||x|| by position is written too (and *pinv_done set).
lsh_status launch_hash_tc(const Dims& D, const Layout& L, const void* x, const void* R,
                          int32_t* buckets, void* ws, cudaStream_t st, void* const* ev,
                          int32_t* hist = nullptr, bool* hist_done = nullptr,
                          float* pinv = nullptr, bool* pinv_done = nullptr) {
  const HashTcPlan p = hash_tc_plan(D.d, D.nb, D.rounds);
  lsh_status s;
  if (hist_done) *hist_done = false;
  if (pinv_done) *pinv_done = false;
  if (p.group == 0) {
    if ((s = mark(ev, 1, st)) != LSH_OK) return s;
    if ((s = launch_hash_exact(D, x, R, buckets, st, true)) != LSH_OK) return s;
    if ((s = mark(ev, 2, st)) != LSH_OK) return s;
    return mark(ev, 3, st);
  }
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  __nv_bfloat16* rt = at<__nv_bfloat16>(ws, L.rt);
  uint64_t* refine = at<uint64_t>(ws, L.refine);
  const int rows_per_round = p.ch * p.nc;
  dim3 pg((rows_per_round + kPrepCols - 1) / kPrepCols, D.rounds);
  k_hash_prep<<<pg, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(R), rt, hdr->pad, D.d, p.half,
                                  rows_per_round);
  if ((s = mark(ev, 1, st)) != LSH_OK) return s;
  CUtensorMap tmx, tmr;
  if (!make_tmap_bf16_2d(&tmx, x, D.d, (uint64_t)D.BH * D.n, (uint64_t)D.d * 2, 64, kHashTile) ||
      !make_tmap_bf16_2d(&tmr, rt, D.d, (uint64_t)D.rounds * rows_per_round, (uint64_t)D.d * 2, 64,
                         p.nc))
    return LSH_ERR_CUDA;
  HashTcArgs a;
  a.buckets = buckets;
  a.refine = refine;
  a.cap = D.BH * D.n;
  a.hdr = hdr;
  a.n = D.n;
  a.nb = D.nb;
  a.rounds = D.rounds;
  a.tiles_per_seq = (D.n + kHashTile - 1) / kHashTile;
  a.tiles = (int)(D.BH * a.tiles_per_seq);
  a.hist = hist;
  a.pinv = pinv;
  a.sort_tile = sort_tile(D.nb);
  a.sort_tiles = D.tiles;
  if (hist != nullptr &&
      cudaMemsetAsync(hist, 0, sizeof(int32_t) * (size_t)D.S * D.nb * D.tiles, st) != cudaSuccess)
    return LSH_ERR_CUDA;
  const int sms = sm_count();
  int per = sms / p.groups;
  if (per < 1) per = 1;
  if (per > a.tiles) per = a.tiles;
  a.ctas_per_group = per;
  const unsigned grid = (unsigned)(per * p.groups);
  auto kern = D.d == 64 ? (p.upw ? k_hash_tc<64, true> : k_hash_tc<64, false>)
                        : (p.upw ? k_hash_tc<128, true> : k_hash_tc<128, false>);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem) !=
      cudaSuccess)
    return LSH_ERR_CUDA;
  kern<<<grid, kHashWarps * 32, p.smem, st>>>(tmx, tmr, a, p);
  if ((s = mark(ev, 2, st)) != LSH_OK) return s;
  // eight CTAs per SM over the rounds: a round's queue (a fraction of a percent
  // of its tokens) is one wave of 8-token batches; surplus CTAs exit at once
  dim3 rg((unsigned)((8 * sms + D.rounds - 1) / D.rounds), D.rounds);
  if (D.d == 64)
    k_hash_refine<64><<<rg, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(x), rt, refine, a.cap,
                                          buckets, D.n, D.nb, D.rounds, rows_per_round, hdr, hist,
                                          a.sort_tile, a.sort_tiles);
  else
    k_hash_refine<128><<<rg, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(x), rt, refine,
                                           a.cap, buckets, D.n, D.nb, D.rounds, rows_per_round,
                                           hdr, hist, a.sort_tile, a.sort_tiles);
  if ((s = last_cuda()) != LSH_OK) return s;
  if (hist_done) *hist_done = hist != nullptr;
  if (pinv_done) *pinv_done = pinv != nullptr;
  return mark(ev, 3, st);
}

lsh_status launch_hash(const Dims& D, const Layout& L, const void* x, const void* R,
                       int32_t* buckets, void* ws, cudaStream_t st, void* const* ev = nullptr,
                       int32_t* hist = nullptr, bool* hist_done = nullptr,
                       float* pinv = nullptr, bool* pinv_done = nullptr) {
  if (D.dtype == LSH_BF16)
    return launch_hash_tc(D, L, x, R, buckets, ws, st, ev, hist, hist_done, pinv, pinv_done);
  if (hist_done) *hist_done = false;
  if (pinv_done) *pinv_done = false;
  lsh_status s;
  if ((s = mark(ev, 1, st)) != LSH_OK) return s;
  if ((s = launch_hash_exact(D, x, R, buckets, st, false)) != LSH_OK) return s;
  if ((s = mark(ev, 2, st)) != LSH_OK) return s;
  return mark(ev, 3, st);
}

template <typename T>
lsh_status launch_sort(const Dims& D, const int32_t* buckets, const void* x, const void* v,
                       int32_t* perm, int32_t* inv, void* xs, void* vs, float* invnorm,
                       int32_t* hist, WsHeader* hdr, cudaStream_t st, void* const* ev = nullptr,
                       bool hist_ready = false) {
  lsh_status s;
  const int tile = sort_tile(D.nb);
  dim3 grid(D.tiles, (unsigned)D.S);
  if (!hist_ready)  // else the hash has counted them
    k_sort_hist<<<grid, 256, sizeof(int32_t) * D.nb, st>>>(buckets, D.n, D.nb, tile, D.tiles,
                                                           hist, hdr);
  if ((s = mark(ev, 4, st)) != LSH_OK) return s;
  k_sort_scan<<<(unsigned)D.S, 1024, 0, st>>>(hist, D.nb * D.tiles);
  if ((s = mark(ev, 5, st)) != LSH_OK) return s;
  {  // stable ranks: perm and inv
    const int nw = sort_warps(D.nb);
    const size_t smem = sort_rank_smem(D.nb);
    if (cudaFuncSetAttribute(k_sort_rank, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return LSH_ERR_CUDA;
    k_sort_rank<<<grid, nw * 32, smem, st>>>(buckets, hist, perm, inv, D.n, D.nb, D.tiles);
  }
  if ((s = last_cuda()) != LSH_OK) return s;
  if ((s = mark(ev, 6, st)) != LSH_OK) return s;
  if (xs != nullptr) {  // the rows in slot order, with 1/||x||
    const int64_t blocks =
        D.BH * (int64_t)((D.n + kGatherSlots - 1) / kGatherSlots) * D.rounds;
    if (blocks > INT32_MAX) return LSH_ERR_UNSUPPORTED;
    auto kern = D.d == 64 ? k_gather_rows<T, 64> : k_gather_rows<T, 128>;
    kern<<<(unsigned)blocks, kGatherWarps * 32, 0, st>>>(
        perm, static_cast<const T*>(x), static_cast<const T*>(v), static_cast<T*>(xs),
        static_cast<T*>(vs), invnorm, D.n, D.rounds);
  }
  return last_cuda();
}

template <typename T, int DD, int QPW>
lsh_status launch_attn_simt_q(const Dims& D, const void* xs, const void* vs, const int32_t* perm,
                              const float* invnorm, T* out_s, float* lse_s, cudaStream_t st) {
  const size_t smem = attn_simt_smem(DD);
  auto kern = k_attn_simt<T, DD, QPW>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSH_ERR_CUDA;
  dim3 grid(D.n / D.m, (unsigned)D.S);
  kern<<<grid, kSimtWarps * 32, smem, st>>>(static_cast<const T*>(xs), static_cast<const T*>(vs),
                                             perm, invnorm, out_s, lse_s, D.n, D.m, D.causal);
  return last_cuda();
}

template <typename T, int DD>
lsh_status launch_attn_simt(const Dims& D, const void* xs, const void* vs, const int32_t* perm,
                            const float* invnorm, T* out_s, float* lse_s, cudaStream_t st) {
  if (D.m <= 16) return launch_attn_simt_q<T, DD, 2>(D, xs, vs, perm, invnorm, out_s, lse_s, st);
  if (D.m <= 32) return launch_attn_simt_q<T, DD, 4>(D, xs, vs, perm, invnorm, out_s, lse_s, st);
  if (D.m <= 64) return launch_attn_simt_q<T, DD, 8>(D, xs, vs, perm, invnorm, out_s, lse_s, st);
  return launch_attn_simt_q<T, DD, 16>(D, xs, vs, perm, invnorm, out_s, lse_s, st);
}

template <int DD, bool CAUSAL>
lsh_status launch_attn_tc_k(const CUtensorMap& tmo, const AttnTcArgs& a, unsigned grid,
                            size_t smem, cudaStream_t st) {
  auto kern = k_attn_tc<DD, CAUSAL>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSH_ERR_CUDA;
  kern<<<grid, kAttnWarps * 32, smem, st>>>(tmo, a);
  return last_cuda();
}

// Chunk attention on the tensor cores, rows of x and v read by perm.
lsh_status launch_attn_tc(const Dims& D, const void* x, const void* v, const int32_t* perm,
                          const float* pinv, void* out_r, float* lse, WsHeader* hdr,
                          cudaStream_t st) {
  CUtensorMap tmo;  // each round's output rows, 32-row stores
  const uint64_t rows = (uint64_t)D.S * D.n;
  if (!make_tmap_bf16_2d(&tmo, out_r, D.d, rows, (uint64_t)D.d * 2, 64, 32)) return LSH_ERR_CUDA;
  AttnTcArgs a;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.pinv = pinv;
  a.perm = perm;
  a.lse = lse;
  a.hdr = hdr;
  a.n = D.n;
  a.rounds = D.rounds;
  a.pairs_per_seg = (D.n / kAttnM + 1) / 2;
  a.units = (int)(D.S * a.pairs_per_seg);  // < 2^31: S x n < 2^31 (attn_tc_supported)
  const unsigned grid = (unsigned)std::min<int64_t>(a.units, sm_count());
  const size_t smem = attn_tc_smem(D.d);
  if (D.d == 64)
    return D.causal ? launch_attn_tc_k<64, true>(tmo, a, grid, smem, st)
                    : launch_attn_tc_k<64, false>(tmo, a, grid, smem, st);
  return D.causal ? launch_attn_tc_k<128, true>(tmo, a, grid, smem, st)
                  : launch_attn_tc_k<128, false>(tmo, a, grid, smem, st);
}

// 1/||x|| by position, when the hash has not written it.
lsh_status launch_row_invnorm(const Dims& D, const void* x, float* pinv, cudaStream_t st) {
  const int64_t rows = D.BH * D.n;
  const int per_block = 256 / kNormParts;
  const unsigned blocks =
      (unsigned)std::min<int64_t>((rows + per_block - 1) / per_block, (int64_t)8 * sm_count());
  if (D.d == 64)
    k_row_invnorm<64><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), pinv, rows);
  else
    k_row_invnorm<128><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), pinv, rows);
  return last_cuda();
}

template <typename T, int DD>
lsh_status launch_merge(const Dims& D, const int32_t* inv, const float* lse, const T* out_r,
                        void* out, cudaStream_t st) {
  const int64_t total = D.BH * D.n;
  const int64_t per_block = kMergeWarps * 32 / (DD * (int)sizeof(T) / 16);  // positions
  const int64_t cap = (int64_t)kMergeCtasPerSm * sm_count();
  const unsigned blocks = (unsigned)std::min<int64_t>((total + per_block - 1) / per_block, cap);
  k_merge<T, DD><<<blocks, kMergeWarps * 32, 0, st>>>(inv, lse, out_r, static_cast<T*>(out), D.n,
                                                        D.rounds, total);
  return last_cuda();
}

template <typename T>
lsh_status forward_typed(const Dims& D, const Layout& L, const void* x, const void* v,
                         const void* R, const int32_t* buckets, void* out, float* lse, void* ws,
                         cudaStream_t st, void* const* ev) {
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  const bool tc = attn_tc_supported(D);
  float* pinv = tc ? at<float>(ws, L.pinv) : nullptr;
  lsh_status s;
  if ((s = mark(ev, 0, st)) != LSH_OK) return s;
  bool hist_ready = false, pinv_ready = false;
  if (!buckets) {
    int32_t* bk = at<int32_t>(ws, L.buckets);
    if ((s = launch_hash(D, L, x, R, bk, ws, st, ev, at<int32_t>(ws, L.hist), &hist_ready, pinv,
                         &pinv_ready)) != LSH_OK)
      return s;
    buckets = bk;
  } else {
    for (int i = 1; i <= 3; ++i)
      if ((s = mark(ev, i, st)) != LSH_OK) return s;
  }
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  T* out_r = at<T>(ws, L.out_s);  // each round's output rows, slot order
  if (tc) {
    // ranks only; the attention reads the rows by perm (and the key scales
    // by position: from the hash, or from the norm pass here)
    if ((s = launch_sort<T>(D, buckets, x, v, perm, inv, nullptr, nullptr, nullptr,
                            at<int32_t>(ws, L.hist), hdr, st, ev, hist_ready)) != LSH_OK)
      return s;
    if (!pinv_ready && (s = launch_row_invnorm(D, x, pinv, st)) != LSH_OK) return s;
    if ((s = mark(ev, 7, st)) != LSH_OK) return s;
    s = launch_attn_tc(D, x, v, perm, pinv, out_r, lse, hdr, st);
  } else {
    float* invnorm = at<float>(ws, L.invnorm);
    void* xs = at<unsigned char>(ws, L.xs);
    void* vs = at<unsigned char>(ws, L.vs);
    if ((s = launch_sort<T>(D, buckets, x, v, perm, inv, xs, vs, invnorm,
                            at<int32_t>(ws, L.hist), hdr, st, ev, hist_ready)) != LSH_OK)
      return s;
    if ((s = mark(ev, 7, st)) != LSH_OK) return s;
    s = D.d == 64 ? launch_attn_simt<T, 64>(D, xs, vs, perm, invnorm, out_r, lse, st)
                  : launch_attn_simt<T, 128>(D, xs, vs, perm, invnorm, out_r, lse, st);
  }
  if (s != LSH_OK) return s;
  if ((s = mark(ev, 8, st)) != LSH_OK) return s;
  s = D.d == 64 ? launch_merge<T, 64>(D, inv, lse, out_r, out, st)
                : launch_merge<T, 128>(D, inv, lse, out_r, out, st);
  if (s != LSH_OK) return s;
  return mark(ev, 9, st);
}

// ---------------------------------------------------------------- dense
struct DenseDims {
  int n, d, causal, qtiles, kstride;
  int64_t BH;
  size_t kscale, queue, total;  // workspace layout
};

lsh_status check_dense(const lsh_attn_desc* desc, DenseDims* D) {
  if (!desc) return LSH_ERR_INVALID_ARG;
  const lsh_attn_desc& q = *desc;
  if (q.batch < 1 || q.heads < 1 || q.n < 1 || q.d < 1 || (q.causal != 0 && q.causal != 1) ||
      (q.dtype != LSH_F32 && q.dtype != LSH_BF16))
    return LSH_ERR_INVALID_ARG;
  if (q.dtype != LSH_BF16 || (q.d != 64 && q.d != 128)) return LSH_ERR_UNSUPPORTED;
  D->n = q.n;
  D->d = q.d;
  D->causal = q.causal;
  D->BH = (int64_t)q.batch * q.heads;
  D->qtiles = (q.n + kDenseTile - 1) / kDenseTile;
  D->kstride = D->qtiles * kDenseTile;
  if (D->BH * D->kstride >= (int64_t(1) << 31)) return LSH_ERR_UNSUPPORTED;
  if (D->BH > 65535) return LSH_ERR_UNSUPPORTED;  // TMA outer coordinate
  size_t off = align_up(sizeof(WsHeader), 256);
  D->kscale = off;
  off = align_up(off + (size_t)D->BH * D->kstride * 4, 256);
  D->queue = off;
  off = align_up(off + (size_t)D->BH * q.n * 4, 256);
  D->total = off;
  return LSH_OK;
}

template <int DD, bool CAUSAL>
lsh_status launch_dense(const DenseDims& D, const void* x, const void* v, void* out, float* lse,
                        void* ws, cudaStream_t st) {
  constexpr int NST = DD == 64 ? 4 : 2;  // K/V ring depth that fits shared memory
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  float* kscale = at<float>(ws, D.kscale);
  int32_t* queue = at<int32_t>(ws, D.queue);
  const int sms = sm_count();
  {
    const int64_t total = D.BH * D.kstride;
    const int per_block = 256 / (DD / 8);
    const unsigned blocks =
        (unsigned)std::min<int64_t>((total + per_block - 1) / per_block, (int64_t)8 * sms);
    k_dense_kscale<DD><<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), kscale, D.n,
                                               D.kstride, total);
  }
  CUtensorMap tmx, tmv, tmo;
  if (!make_tmap_bf16_3d(&tmx, x, DD, D.n, D.BH, 64, kDenseTile) ||
      !make_tmap_bf16_3d(&tmv, v, DD, D.n, D.BH, 64, kDenseTile) ||
      !make_tmap_bf16_3d(&tmo, out, DD, D.n, D.BH, 64, 32))
    return LSH_ERR_CUDA;
  DenseArgs a;
  a.kscale = kscale;
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.lse = lse;
  a.fix_queue = queue;
  a.hdr = hdr;
  a.n = D.n;
  a.BH = (int)D.BH;
  a.qtiles = D.qtiles;
  a.kstride = D.kstride;
  a.units = D.BH * D.qtiles;
  const unsigned grid = (unsigned)std::min<int64_t>(a.units, sms);
  const size_t smem = dense_smem<DD, NST>();
  auto kern = k_attn_dense<DD, CAUSAL, NST>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSH_ERR_CUDA;
  kern<<<grid, kDenseWarps * 32, smem, st>>>(tmx, tmv, tmo, a);
  // rows queued by the kernel (none for inputs of moderate norm) are redone exactly
  k_dense_fixup<DD, CAUSAL><<<2 * sms, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(v), kscale,
      static_cast<__nv_bfloat16*>(out), lse, queue, hdr, D.n, D.kstride);
  return last_cuda();
}

// ---------------------------------------------------------------- backward
struct BwdLayout {
  size_t header, perm, inv, hist, pinv, pos_tab, qtab, ktab, dq, dxk, dv, total;
};

// Backward support: bf16 and the tensor-core chunk (64), as the forward's
// tensor-core path.
lsh_status check_bwd(const lsh_attn_desc* desc, Dims* D, BwdLayout* L) {
  lsh_status s = check_desc(desc, D, true);
  if (s != LSH_OK) return s;
  if (!attn_tc_supported(*D)) return LSH_ERR_UNSUPPORTED;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t sn = (size_t)D->S * D->n;
  L->header = take(sizeof(WsHeader));
  L->perm = take(sn * 4);
  L->inv = take(sn * 4);
  L->hist = take((size_t)D->S * D->nb * D->tiles * 4);
  L->pinv = take((size_t)D->BH * D->n * 4);
  L->pos_tab = take((size_t)D->BH * D->n * 8);
  L->qtab = take(sn * 16);
  L->ktab = take(sn * 16);
  L->dq = take(sn * D->d * 4);
  L->dxk = take(sn * D->d * 4);
  L->dv = take(sn * D->d * 4);
  L->total = off;
  return LSH_OK;
}

template <int DD, bool CAUSAL>
lsh_status launch_bwd_tc(const BwdArgs& a, const Dims& D, cudaStream_t st) {
  const int sms = sm_count();
  const unsigned grid = (unsigned)std::min<int64_t>(a.units, sms);
  // x, v and g in position order, one-row boxes for the gathers
  CUtensorMap tmx, tmv, tmg;
  const uint64_t prow = (uint64_t)D.BH * D.n;
  if (!make_tmap_bf16_2d(&tmx, a.x, DD, prow, (uint64_t)DD * 2, 64, 1) ||
      !make_tmap_bf16_2d(&tmv, a.v, DD, prow, (uint64_t)DD * 2, 64, 1) ||
      !make_tmap_bf16_2d(&tmg, a.g, DD, prow, (uint64_t)DD * 2, 64, 1))
    return LSH_ERR_CUDA;
  {
    auto kern = k_bwd_dq<DD, CAUSAL>;
    const size_t smem = bwd_dq_smem<DD>();
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return LSH_ERR_CUDA;
    kern<<<grid, kBwdWarps * 32, smem, st>>>(tmx, tmv, tmg, a);
  }
  {
    auto kern = k_bwd_dkv<DD, CAUSAL>;
    const size_t smem = bwd_dkv_smem<DD>();
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return LSH_ERR_CUDA;
    kern<<<grid, kBwdWarps * 32, smem, st>>>(tmx, tmv, tmg, a);
  }
  return last_cuda();
}

template <int DD>
lsh_status backward_d(const Dims& D, const BwdLayout& L, const void* x, const void* v,
                      const int32_t* buckets, const void* out, const float* lse,
                      const void* dout, const float* dlse, void* dx, void* dv, void* ws,
                      cudaStream_t st) {
  using T = __nv_bfloat16;
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* inv = at<int32_t>(ws, L.inv);
  lsh_status s = launch_sort<T>(D, buckets, x, v, perm, inv, nullptr, nullptr, nullptr,
                                at<int32_t>(ws, L.hist), hdr, st);
  if (s != LSH_OK) return s;
  float* pinv = at<float>(ws, L.pinv);
  if ((s = launch_row_invnorm(D, x, pinv, st)) != LSH_OK) return s;
  const int sms = sm_count();
  const int64_t pos_total = D.BH * D.n;
  float2* pos_tab = at<float2>(ws, L.pos_tab);
  const int64_t pos_per_block = 8 * (32 / (DD * (int)sizeof(T) / 16));
  k_bwd_prep_pos<T, DD><<<(unsigned)std::min<int64_t>((pos_total + pos_per_block - 1) / pos_per_block,
                                                      8 * sms),
                          256, 0, st>>>(
      lse, static_cast<const T*>(out), static_cast<const T*>(dout), pos_tab, D.n, D.rounds,
      pos_total);
  const int64_t slot_total = D.S * D.n;
  float4* qtab = at<float4>(ws, L.qtab);
  float4* ktab = at<float4>(ws, L.ktab);
  k_bwd_prep_slot<<<(unsigned)std::min<int64_t>((slot_total + 255) / 256, 8 * sms), 256, 0, st>>>(
      perm, lse, dlse, pos_tab, pinv, qtab, ktab, D.n, D.rounds, 1.0f / sqrtf((float)DD),
      slot_total);
  BwdArgs a;
  a.x = static_cast<const T*>(x);
  a.v = static_cast<const T*>(v);
  a.g = static_cast<const T*>(dout);
  a.qtab = qtab;
  a.ktab = ktab;
  a.dq = at<float>(ws, L.dq);
  a.dxk = at<float>(ws, L.dxk);
  a.dv = at<float>(ws, L.dv);
  a.hdr = hdr;
  a.n = D.n;
  a.rounds = D.rounds;
  a.pairs_per_seg = (D.n / kAttnM + 1) / 2;
  a.units = D.S * a.pairs_per_seg;
  a.oob = (int)(D.BH * D.n);
  if ((s = D.causal ? launch_bwd_tc<DD, true>(a, D, st) : launch_bwd_tc<DD, false>(a, D, st)) !=
      LSH_OK)
    return s;
  k_bwd_unsort<T, DD><<<(unsigned)std::min<int64_t>((pos_total + 7) / 8, 8 * sms), 256, 0, st>>>(
      inv, a.dq, a.dxk, a.dv, static_cast<T*>(dx), static_cast<T*>(dv), D.n, D.rounds, pos_total);
  return last_cuda();
}

// ---------------------------------------------------------------- top-k variant
struct TopkLayout {
  size_t header, bucket, perm, inv, hist, cand, total;
};

lsh_status check_topk(const lsh_topk_desc* t, Dims* D, TopkLayout* L) {
  if (!t) return LSH_ERR_INVALID_ARG;
  const lsh_topk_desc& q = *t;
  if (q.batch < 1 || q.heads < 1 || q.n < 1 || q.d < 1 || q.n_buckets < 1 || q.n_bits < 1 ||
      q.top_k < 1 || q.rounds < 1 || (q.causal != 0 && q.causal != 1))
    return LSH_ERR_INVALID_ARG;
  if ((q.d != 64 && q.d != 128) || q.n_bits > kTopkMaxBits || q.top_k > kTopkMaxK ||
      q.rounds > kTopkMaxRounds)
    return LSH_ERR_UNSUPPORTED;
  // the counting sort takes an even bucket count in [2, 4096]
  const lsh_attn_desc ad{q.batch, q.heads, q.n, q.d, q.n_buckets, 1, q.rounds, q.causal, LSH_BF16};
  lsh_status s = check_desc(&ad, D, false);
  if (s != LSH_OK) return s;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  const size_t sn = (size_t)D->S * D->n;
  L->header = take(sizeof(WsHeader));
  L->bucket = take(sn * 4);
  L->perm = take(sn * 4);
  L->inv = take(sn * 4);
  L->hist = take((size_t)D->S * D->nb * D->tiles * 4);
  L->cand = take(sn * q.top_k * 4);
  L->total = off;
  return LSH_OK;
}

template <int DD>
lsh_status topk_forward_d(const Dims& D, const TopkLayout& L, const lsh_topk_desc& q,
                          const void* x, const void* v, const void* proj, void* out, float* lse,
                          int32_t* cand, void* ws, cudaStream_t st) {
  using T = __nv_bfloat16;
  const int sms = sm_count();
  int32_t* bucket = at<int32_t>(ws, L.bucket);
  int32_t* perm = at<int32_t>(ws, L.perm);
  const int64_t hash_total = D.S * D.n;
  k_tk_hash<DD><<<(unsigned)std::min<int64_t>((hash_total + 255) / 256, 16 * sms), 256, 0, st>>>(
      static_cast<const T*>(x), static_cast<const T*>(proj), bucket, D.n, D.rounds, q.n_bits,
      q.n_buckets, hash_total);
  lsh_status s = launch_sort<T>(D, bucket, x, v, perm, at<int32_t>(ws, L.inv), nullptr, nullptr,
                                nullptr, at<int32_t>(ws, L.hist), at<WsHeader>(ws, L.header), st);
  if (s != LSH_OK) return s;
  const int64_t sel_total = D.S * D.n;  // warps
  k_tk_select<DD><<<(unsigned)std::min<int64_t>((sel_total + 7) / 8, 16 * sms), 256, 0, st>>>(
      static_cast<const T*>(x), bucket, perm, cand, D.n, D.rounds, q.top_k, q.causal, sel_total);
  const int64_t att_total = D.BH * D.n;
  k_tk_attend<DD><<<(unsigned)std::min<int64_t>((att_total + 7) / 8, 16 * sms), 256, 0, st>>>(
      static_cast<const T*>(x), static_cast<const T*>(v), cand, static_cast<T*>(out), lse, D.n,
      D.rounds, q.top_k, att_total);
  return last_cuda();
}

}  // namespace

// ------------------------------------------------------------------ C ABI
extern "C" {

const char* lsh_attn_status_string(lsh_status s) {
  switch (s) {
    case LSH_OK: return "LSH_OK";
    case LSH_ERR_INVALID_ARG: return "LSH_ERR_INVALID_ARG: invalid argument";
    case LSH_ERR_UNSUPPORTED: return "LSH_ERR_UNSUPPORTED: problem outside the supported set";
    case LSH_ERR_WORKSPACE: return "LSH_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case LSH_ERR_CUDA: return "LSH_ERR_CUDA: a CUDA runtime call failed";
    case LSH_ERR_TIMEOUT: return "LSH_ERR_TIMEOUT: a bounded wait in a kernel gave up";
    case LSH_ERR_DEVICE: return "LSH_ERR_DEVICE: a kernel rejected its input";
  }
  return "unknown lsh_status";
}

lsh_status lsh_attn_workspace_size(const lsh_attn_desc* desc, size_t* bytes) {
  Dims D;
  lsh_status s = check_desc(desc, &D, true);
  if (s != LSH_OK) return s;
  if (!bytes) return LSH_ERR_INVALID_ARG;
  *bytes = layout_of(D).total;
  return LSH_OK;
}

lsh_status lsh_attn_hash(const lsh_attn_desc* desc, const void* x, const void* R,
                         int32_t* buckets, void* ws, size_t ws_bytes, void* stream) {
  Dims D;
  Layout L;
  lsh_status s = check_desc(desc, &D, false);
  if (s != LSH_OK) return s;
  if (!x || !R || !buckets) return LSH_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(R)) return LSH_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes, &L)) != LSH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  return launch_hash(D, L, x, R, buckets, ws, st);
}

lsh_status lsh_attn_sort(const lsh_attn_desc* desc, const int32_t* buckets, const void* x,
                         const void* v, int32_t* perm, void* xs, void* vs, void* ws,
                         size_t ws_bytes, void* stream) {
  Dims D;
  Layout L;
  lsh_status s = check_desc(desc, &D, false);
  if (s != LSH_OK) return s;
  if (!buckets || !perm) return LSH_ERR_INVALID_ARG;
  const bool gather = x || v || xs || vs;
  if (gather && (!x || !v || !xs || !vs)) return LSH_ERR_INVALID_ARG;
  if (gather && !(aligned16(x) && aligned16(v) && aligned16(xs) && aligned16(vs)))
    return LSH_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes, &L)) != LSH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  int32_t* inv = at<int32_t>(ws, L.inv);
  float* invnorm = at<float>(ws, L.invnorm);
  int32_t* hist = at<int32_t>(ws, L.hist);
  if (D.dtype == LSH_BF16)
    return launch_sort<__nv_bfloat16>(D, buckets, x, v, perm, inv, gather ? xs : nullptr,
                                      gather ? vs : nullptr, invnorm, hist, hdr, st);
  return launch_sort<float>(D, buckets, x, v, perm, inv, gather ? xs : nullptr,
                            gather ? vs : nullptr, invnorm, hist, hdr, st);
}

lsh_status lsh_attn_forward(const lsh_attn_desc* desc, const void* x, const void* v,
                            const void* R, const int32_t* buckets, void* out, float* lse,
                            void* ws, size_t ws_bytes, void* stream) {
  return lsh_attn_forward_profiled(desc, x, v, R, buckets, out, lse, ws, ws_bytes, stream,
                                   nullptr);
}

lsh_status lsh_attn_forward_profiled(const lsh_attn_desc* desc, const void* x, const void* v,
                                     const void* R, const int32_t* buckets, void* out, float* lse,
                                     void* ws, size_t ws_bytes, void* stream,
                                     void* const* events) {
  Dims D;
  Layout L;
  lsh_status s = check_desc(desc, &D, true);
  if (s != LSH_OK) return s;
  if (!x || !v || !out || !lse || (!buckets && !R)) return LSH_ERR_INVALID_ARG;
  if (!(aligned16(x) && aligned16(v) && aligned16(out))) return LSH_ERR_INVALID_ARG;
  if (!buckets && !aligned16(R)) return LSH_ERR_INVALID_ARG;
  if ((s = check_ws(D, ws, ws_bytes, &L)) != LSH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  return D.dtype == LSH_BF16
             ? forward_typed<__nv_bfloat16>(D, L, x, v, R, buckets, out, lse, ws, st, events)
             : forward_typed<float>(D, L, x, v, R, buckets, out, lse, ws, st, events);
}

lsh_status lsh_attn_dense_workspace_size(const lsh_attn_desc* desc, size_t* bytes) {
  DenseDims D;
  lsh_status s = check_dense(desc, &D);
  if (s != LSH_OK) return s;
  if (!bytes) return LSH_ERR_INVALID_ARG;
  *bytes = D.total;
  return LSH_OK;
}

lsh_status lsh_attn_dense_forward(const lsh_attn_desc* desc, const void* x, const void* v,
                                  void* out, float* lse, void* ws, size_t ws_bytes,
                                  void* stream) {
  DenseDims D;
  lsh_status s = check_dense(desc, &D);
  if (s != LSH_OK) return s;
  if (!x || !v || !out || !lse) return LSH_ERR_INVALID_ARG;
  if (!(aligned16(x) && aligned16(v) && aligned16(out))) return LSH_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255) != 0 || ws_bytes < D.total) return LSH_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  if (D.d == 64)
    return D.causal ? launch_dense<64, true>(D, x, v, out, lse, ws, st)
                    : launch_dense<64, false>(D, x, v, out, lse, ws, st);
  return D.causal ? launch_dense<128, true>(D, x, v, out, lse, ws, st)
                  : launch_dense<128, false>(D, x, v, out, lse, ws, st);
}

lsh_status lsh_attn_backward_workspace_size(const lsh_attn_desc* desc, size_t* bytes) {
  Dims D;
  BwdLayout L;
  lsh_status s = check_bwd(desc, &D, &L);
  if (s != LSH_OK) return s;
  if (!bytes) return LSH_ERR_INVALID_ARG;
  *bytes = L.total;
  return LSH_OK;
}

lsh_status lsh_attn_backward(const lsh_attn_desc* desc, const void* x, const void* v,
                             const int32_t* buckets, const void* out, const float* lse,
                             const void* dout, const float* dlse, void* dx, void* dv, void* ws,
                             size_t ws_bytes, void* stream) {
  Dims D;
  BwdLayout L;
  lsh_status s = check_bwd(desc, &D, &L);
  if (s != LSH_OK) return s;
  if (!x || !v || !buckets || !out || !lse || !dout || !dx || !dv) return LSH_ERR_INVALID_ARG;
  if (!(aligned16(x) && aligned16(v) && aligned16(out) && aligned16(dout) && aligned16(dx) &&
        aligned16(dv)))
    return LSH_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255) != 0 || ws_bytes < L.total) return LSH_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  return D.d == 64 ? backward_d<64>(D, L, x, v, buckets, out, lse, dout, dlse, dx, dv, ws, st)
                   : backward_d<128>(D, L, x, v, buckets, out, lse, dout, dlse, dx, dv, ws, st);
}

lsh_status lsh_topk_workspace_size(const lsh_topk_desc* desc, size_t* bytes) {
  Dims D;
  TopkLayout L;
  lsh_status s = check_topk(desc, &D, &L);
  if (s != LSH_OK) return s;
  if (!bytes) return LSH_ERR_INVALID_ARG;
  *bytes = L.total;
  return LSH_OK;
}

lsh_status lsh_topk_forward(const lsh_topk_desc* desc, const void* x, const void* v,
                            const void* proj, void* out, float* lse, int32_t* cand, void* ws,
                            size_t ws_bytes, void* stream) {
  Dims D;
  TopkLayout L;
  lsh_status s = check_topk(desc, &D, &L);
  if (s != LSH_OK) return s;
  if (!x || !v || !proj || !out || !lse) return LSH_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255) != 0 || ws_bytes < L.total) return LSH_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = reset_header(ws, st)) != LSH_OK) return s;
  int32_t* c = cand ? cand : at<int32_t>(ws, L.cand);
  return D.d == 64 ? topk_forward_d<64>(D, L, *desc, x, v, proj, out, lse, c, ws, st)
                   : topk_forward_d<128>(D, L, *desc, x, v, proj, out, lse, c, ws, st);
}

lsh_status lsh_attn_get_diag(const void* ws, void* stream, lsh_attn_diag* diag) {
  if (!ws || !diag) return LSH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return LSH_ERR_CUDA;
  WsHeader h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return LSH_ERR_CUDA;
  diag->status = h.status;
  diag->hash_refined = h.hash_refined;
  diag->bad_bucket_ids = h.bad_bucket_ids;
  diag->reserved = 0;
  return LSH_OK;
}

lsh_status lsh_attn_selftest_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us,
                                          void* stream) {
  if (!ws || ws_bytes < sizeof(WsHeader) || limit_us < 1 || limit_us > 2000000u)
    return LSH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  lsh_status s = reset_header(ws, st);
  if (s != LSH_OK) return s;
  k_wait_selftest<<<1, 32, 0, st>>>(static_cast<WsHeader*>(ws), (uint64_t)limit_us * 1000u);
  return last_cuda();
}

lsh_status lsh_attn_get_device_status(const void* ws, void* stream) {
  lsh_attn_diag d;
  lsh_status s = lsh_attn_get_diag(ws, stream, &d);
  if (s != LSH_OK) return s;
  return static_cast<lsh_status>(d.status);
}

}  // extern "C"
