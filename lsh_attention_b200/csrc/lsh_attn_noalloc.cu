// lsh_attn_sort_noalloc: the stable bucket sort of lsh_attn_sort for callers
// that must not allocate device memory and cannot hand over a workspace.
//
// Some callers cannot call cudaMalloc: a plug-in hosted by a runtime that owns
// every byte of device memory and forbids allocations outside its own arena,
// or a latency-critical loop where cudaMalloc / cudaFree would synchronise the
// device. This entry point takes only the inputs and the output; its scratch
// (status header, bucket histograms, inverse permutation) is a fixed array in
// the library's own device memory, which every GPU that loads the library
// holds until the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "lsh_attn.h"
// This file is a translation unit of its own: the sort kernels get file-local
// names so they do not collide with lsh_attn.cu's.
#define k_sort_hist k_sort_hist_noalloc
#define k_sort_scan k_sort_scan_noalloc
#define k_sort_rank k_sort_rank_noalloc
#include "sort.cuh"
#undef k_sort_hist
#undef k_sort_scan
#undef k_sort_rank

namespace {

using namespace lsh;

// The scratch. Its size is LSH_ATTN_NOALLOC_SCRATCH_BYTES.
static __device__ __align__(256) unsigned char g_sort_scratch[LSH_ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
lsh_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LSH_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sort_scratch) != cudaSuccess || p == nullptr)
      return LSH_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LSH_OK;
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

extern "C" lsh_status lsh_attn_sort_noalloc(const lsh_attn_desc* desc, const int32_t* buckets,
                                            int32_t* perm, void* stream) {
  if (!desc || !buckets || !perm) return LSH_ERR_INVALID_ARG;
  const lsh_attn_desc& q = *desc;
  if (q.batch < 1 || q.heads < 1 || q.n < 1 || q.n_buckets < 1 || q.rounds < 1)
    return LSH_ERR_INVALID_ARG;
  if (q.n_buckets % 2 != 0 || q.n_buckets < 2 || q.n_buckets > 4096 || q.rounds > 16)
    return LSH_ERR_UNSUPPORTED;
  if ((int64_t)q.n * q.n_buckets >= (int64_t(1) << 31)) return LSH_ERR_UNSUPPORTED;
  const int64_t segs = (int64_t)q.batch * q.heads * q.rounds;
  if (segs > 65535) return LSH_ERR_UNSUPPORTED;
  const int tile = sort_tile(q.n_buckets);
  const int tiles = (q.n + tile - 1) / tile;
  // scratch layout: header | histograms [seg][nb][tiles] | inv [seg][n]
  const size_t hdr_bytes = round256(sizeof(WsHeader));
  const size_t hist_bytes = round256((size_t)segs * q.n_buckets * tiles * 4);
  const size_t inv_bytes = (size_t)segs * q.n * 4;
  if (hdr_bytes + hist_bytes + inv_bytes > (size_t)LSH_ATTN_NOALLOC_SCRATCH_BYTES)
    return LSH_ERR_UNSUPPORTED;  // beyond the built-in scratch: use lsh_attn_sort
  void* base = nullptr;
  lsh_status s = scratch_address(&base);
  if (s != LSH_OK) return s;
  unsigned char* b = static_cast<unsigned char*>(base);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(b);
  int32_t* hist = reinterpret_cast<int32_t*>(b + hdr_bytes);
  int32_t* inv = reinterpret_cast<int32_t*>(b + hdr_bytes + hist_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the counters must start at zero; the histograms and inv are fully rewritten
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return LSH_ERR_CUDA;
  dim3 grid(tiles, (unsigned)segs);
  k_sort_hist_noalloc<<<grid, 256, sizeof(int32_t) * q.n_buckets, st>>>(buckets, q.n, q.n_buckets, tile,
                                                                tiles, hist, hdr);
  k_sort_scan_noalloc<<<(unsigned)segs, 1024, 0, st>>>(hist, q.n_buckets * tiles);
  const int nw = sort_warps(q.n_buckets);
  const size_t smem = sort_rank_smem(q.n_buckets);
  if (cudaFuncSetAttribute(k_sort_rank_noalloc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return LSH_ERR_CUDA;
  k_sort_rank_noalloc<<<grid, nw * 32, smem, st>>>(buckets, hist, perm, inv, q.n, q.n_buckets,
                                                   tiles);
  return cudaGetLastError() == cudaSuccess ? LSH_OK : LSH_ERR_CUDA;
}
