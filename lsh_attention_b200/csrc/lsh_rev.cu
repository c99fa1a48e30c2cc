// Host side of the reversible block entry points declared in
// include/lsh_attn.h: a Reformer layer of LSH attention and a chunked
// feed-forward layer joined by reversible residuals ("Reformer: LSH attention
// and reversible layers" (dtcms.com), §二.2 and §二.3):
//   y1 = x1 + Attn(x2),   y2 = x2 + FFN(y1)
//   (inverse)  x2 = y2 - FFN(y1),   x1 = y1 - Attn(x2)
// Attn(x) = heads(LSH attention of (x W_qk^T, x W_v^T)) W_o^T and
// FFN(y) = max(y W1^T + b1, 0) W2^T + b2, the latter one chunk of rows at a
// time. The products run in k_gemm_tc (tcgen05), the attention in the
// library's own forward; nothing here allocates.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "gemm.cuh"
#include "lsh_attn.h"
#include "tma_host.cuh"

namespace {

using namespace lsh;

inline size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct RevLayout {
  size_t header, qk, v, att, lse, hid, bk, attn, total;
  size_t attn_bytes;
  int64_t rows, chunk_rows;
};

lsh_status check_rev(const lsh_rev_desc* r, lsh_attn_desc* ad, RevLayout* L) {
  if (!r) return LSH_ERR_INVALID_ARG;
  const lsh_rev_desc& q = *r;
  if (q.batch < 1 || q.n < 1 || q.heads < 1 || q.d_head < 1 || q.d_model < 1 || q.d_ff < 1 ||
      q.ffn_chunk < 1 || (q.causal != 0 && q.causal != 1))
    return LSH_ERR_INVALID_ARG;
  if (q.d_model != q.heads * q.d_head) return LSH_ERR_INVALID_ARG;
  if (q.n % kGemmBM != 0 || q.d_model % kGemmBN != 0 || q.d_ff % kGemmBN != 0 ||
      q.ffn_chunk % kGemmBM != 0)
    return LSH_ERR_UNSUPPORTED;
  *ad = lsh_attn_desc{q.batch, q.heads, q.n, q.d_head, q.n_buckets, q.chunk, q.rounds, q.causal,
                      LSH_BF16};
  lsh_status s = lsh_attn_workspace_size(ad, &L->attn_bytes);
  if (s != LSH_OK) return s;
  if (q.chunk != 64) return LSH_ERR_UNSUPPORTED;  // the tensor-core attention
  L->rows = (int64_t)q.batch * q.n;
  if (L->rows * std::max(q.d_model, q.d_ff) >= (int64_t(1) << 40)) return LSH_ERR_UNSUPPORTED;
  L->chunk_rows = std::min<int64_t>(q.ffn_chunk, L->rows);
  const size_t act = (size_t)L->rows * q.d_model * 2;
  size_t off = 0;
  auto take = [&](size_t b) {
    const size_t at = off;
    off = align256(off + b);
    return at;
  };
  L->header = take(sizeof(WsHeader));  // the GEMMs' status, and the block's
  L->qk = take(act);
  L->v = take(act);
  L->att = take(act);
  L->lse = take((size_t)q.batch * q.heads * q.rounds * q.n * 4);
  L->hid = take((size_t)L->chunk_rows * q.d_ff * 2);
  L->bk = take((size_t)q.batch * q.heads * q.rounds * q.n * 4);
  L->attn = take(L->attn_bytes);
  L->total = off;
  return LSH_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<unsigned char*>(ws) + off);
}

// C = res + sign * act(A B^T + bias). a_heads / c_heads: A / C in the
// head-split layout [batch][heads][n][d] (rows = batch * n + position).
lsh_status gemm(const void* A, int64_t M, int K, bool a_heads, const void* B, int N, void* C,
                bool c_heads, const float* bias, const void* res, bool relu, float sign,
                const lsh_rev_desc& q, WsHeader* hdr, cudaStream_t st) {
  CUtensorMap ta, tb, tc;
  bool ok = a_heads ? make_tmap_bf16_heads(&ta, A, q.d_head, q.n, q.heads, q.batch, kGemmBK,
                                           kGemmBM)
                    : make_tmap_bf16_2d(&ta, A, K, M, (uint64_t)K * 2, kGemmBK, kGemmBM);
  ok = ok && make_tmap_bf16_2d(&tb, B, K, N, (uint64_t)K * 2, kGemmBK, kGemmBN);
  ok = ok && (c_heads ? make_tmap_bf16_heads(&tc, C, q.d_head, q.n, q.heads, q.batch, 64, 32)
                      : make_tmap_bf16_2d(&tc, C, N, M, (uint64_t)N * 2, 64, 32));
  if (!ok) return LSH_ERR_CUDA;
  GemmArgs g;
  g.bias = bias;
  g.res = static_cast<const __nv_bfloat16*>(res);
  g.M = (int)M;
  g.N = N;
  g.K = K;
  g.relu = relu ? 1 : 0;
  g.sign = sign;
  g.a_split_n = a_heads ? q.n : 0;
  g.a_split_d = a_heads ? q.d_head : 0;
  g.c_split_n = c_heads ? q.n : 0;
  g.c_split_d = c_heads ? q.d_head : 0;
  g.hdr = hdr;
  const int tiles = (int)((M + kGemmBM - 1) / kGemmBM) * ((N + kGemmBN - 1) / kGemmBN);
  const size_t smem = gemm_smem();
  if (cudaFuncSetAttribute(k_gemm_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LSH_ERR_CUDA;
  k_gemm_tc<<<std::min(tiles, sm_count()), kGemmWarps * 32, smem, st>>>(ta, tb, tc, g);
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

// out = res + sign * Attn(x); the bucket ids are hashed into bk first when
// `hash` is set (from this x's projection), else read from bk.
lsh_status attention_layer(const lsh_rev_desc& q, const lsh_attn_desc& ad, const RevLayout& L,
                           const void* x, const void* w_qk, const void* w_v, const void* w_o,
                           const void* R, int32_t* bk, bool hash, const void* res, float sign,
                           void* out, void* ws, cudaStream_t st) {
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  void* qk = at<unsigned char>(ws, L.qk);
  void* v = at<unsigned char>(ws, L.v);
  void* att = at<unsigned char>(ws, L.att);
  lsh_status s;
  if ((s = gemm(x, L.rows, q.d_model, false, w_qk, q.d_model, qk, true, nullptr, nullptr, false,
                1.f, q, hdr, st)) != LSH_OK)
    return s;
  if ((s = gemm(x, L.rows, q.d_model, false, w_v, q.d_model, v, true, nullptr, nullptr, false, 1.f,
                q, hdr, st)) != LSH_OK)
    return s;
  void* aws = at<unsigned char>(ws, L.attn);
  if (hash && (s = lsh_attn_hash(&ad, qk, R, bk, aws, L.attn_bytes, st)) != LSH_OK) return s;
  if ((s = lsh_attn_forward(&ad, qk, v, nullptr, bk, att, at<float>(ws, L.lse), aws,
                            L.attn_bytes, st)) != LSH_OK)
    return s;
  return gemm(att, L.rows, q.d_model, true, w_o, q.d_model, out, false, nullptr, res, false, sign,
              q, hdr, st);
}

// out = res + sign * FFN(y), one chunk of rows at a time.
lsh_status ffn_layer(const lsh_rev_desc& q, const RevLayout& L, const void* y, const void* w1,
                     const float* b1, const void* w2, const float* b2, const void* res,
                     float sign, void* out, void* ws, cudaStream_t st) {
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  void* hid = at<unsigned char>(ws, L.hid);
  for (int64_t r0 = 0; r0 < L.rows; r0 += L.chunk_rows) {
    const int64_t rows = std::min(L.chunk_rows, L.rows - r0);
    const size_t o = (size_t)r0 * q.d_model * 2;
    lsh_status s = gemm(static_cast<const unsigned char*>(y) + o, rows, q.d_model, false, w1,
                        q.d_ff, hid, false, b1, nullptr, true, 1.f, q, hdr, st);
    if (s != LSH_OK) return s;
    s = gemm(hid, rows, q.d_ff, false, w2, q.d_model, static_cast<unsigned char*>(out) + o, false,
             b2, static_cast<const unsigned char*>(res) + o, false, sign, q, hdr, st);
    if (s != LSH_OK) return s;
  }
  return LSH_OK;
}

inline bool a16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// The attention's status (its own workspace header) joins the block's.
__global__ void k_status_merge(WsHeader* dst, const WsHeader* src) {
  if (src->status != 0) record_status(dst, src->status);
}

}  // namespace

extern "C" {

lsh_status lsh_rev_workspace_size(const lsh_rev_desc* desc, size_t* bytes) {
  lsh_attn_desc ad;
  RevLayout L;
  lsh_status s = check_rev(desc, &ad, &L);
  if (s != LSH_OK) return s;
  if (!bytes) return LSH_ERR_INVALID_ARG;
  *bytes = L.total;
  return LSH_OK;
}

lsh_status lsh_rev_block(const lsh_rev_desc* desc, int inverse, const void* in1, const void* in2,
                         const lsh_rev_weights* w, const void* R, int32_t* buckets, void* out1,
                         void* out2, void* ws, size_t ws_bytes, void* stream) {
  lsh_attn_desc ad;
  RevLayout L;
  lsh_status s = check_rev(desc, &ad, &L);
  if (s != LSH_OK) return s;
  if (!in1 || !in2 || !w || !out1 || !out2 || !buckets || !w->w_qk || !w->w_v || !w->w_o ||
      !w->w1 || !w->w2)
    return LSH_ERR_INVALID_ARG;
  const bool hash = !inverse && desc->hash_buckets;
  if (hash && !R) return LSH_ERR_INVALID_ARG;
  const void* ptrs[] = {in1, in2, out1, out2, w->w_qk, w->w_v, w->w_o, w->w1, w->w2};
  for (const void* p : ptrs)
    if (!a16(p)) return LSH_ERR_INVALID_ARG;
  if (hash && !a16(R)) return LSH_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws & 255) != 0 || ws_bytes < L.total) return LSH_ERR_WORKSPACE;
  const lsh_rev_desc& q = *desc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WsHeader* hdr = at<WsHeader>(ws, L.header);
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return LSH_ERR_CUDA;
  if (!inverse) {
    // y1 = x1 + Attn(x2); y2 = x2 + FFN(y1)
    if ((s = attention_layer(q, ad, L, in2, w->w_qk, w->w_v, w->w_o, R, buckets, hash, in1, 1.f,
                             out1, ws, st)) != LSH_OK)
      return s;
    s = ffn_layer(q, L, out1, w->w1, w->b1, w->w2, w->b2, in2, 1.f, out2, ws, st);
  } else {
    // x2 = y2 - FFN(y1); x1 = y1 - Attn(x2), with the forward's bucket ids
    if ((s = ffn_layer(q, L, in1, w->w1, w->b1, w->w2, w->b2, in2, -1.f, out2, ws, st)) != LSH_OK)
      return s;
    s = attention_layer(q, ad, L, out2, w->w_qk, w->w_v, w->w_o, R, buckets, false, in1, -1.f,
                        out1, ws, st);
  }
  if (s != LSH_OK) return s;
  k_status_merge<<<1, 1, 0, st>>>(hdr, at<WsHeader>(ws, L.attn));
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}

}  // extern "C"
