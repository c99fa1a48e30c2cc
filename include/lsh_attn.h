/*
 * lsh_attn.h -- C ABI of the B200 (sm_100a) Reformer shared-QK LSH-attention
 * forward pass.
 *
 * The method (sources are web pages on Reformer, cited by title and section):
 *   - hash: for b buckets a random R of size [dimension, b/2] maps x to
 *     argmax([xR ; -xR])                  ("Reformer summary", §局部敏感哈希)
 *   - several independent hash rounds     ("Reformer summary", §多輪LSH哈希)
 *   - sort the tokens by bucket, then by position; cut the sorted order into
 *     chunks of m and attend inside them  ("Reformer summary", §局部敏感哈希注意力)
 *   - keys are the shared vectors scaled to unit length, logits are scaled by
 *     1/sqrt(d) ("Reformer: LSH attention and reversible layers", §二.1)
 *   - a token attends to itself only when nothing else is available
 *                                         ("Reformer summary", §共享QK中的自掩碼)
 * Readings taken where the pages are silent: a query in chunk c sees the keys
 * of chunks c-1 and c (chunk 0 sees only itself); the self logit is -1e5;
 * causal masking removes keys at later positions; rounds are merged by
 * weighting each round's output with exp(lse_r - logsumexp_r lse_r); argmax
 * ties go to the first index of [xR ; -xR].
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers owned by the caller. The library
 *     never allocates device memory; scratch space is the caller's workspace of
 *     at least lsh_attn_workspace_size() bytes, 256-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronise the host, except
 *     lsh_attn_get_device_status / lsh_attn_get_diag, which synchronise
 *     `stream`.
 *   - Argument errors are detected on the host before anything is launched;
 *     nothing is written then. Errors found by the kernels (a caller bucket id
 *     outside [0, n_buckets), a bounded wait that gave up) are recorded in the
 *     workspace status word and read with lsh_attn_get_device_status.
 *   - Results are deterministic: identical inputs give bit-identical outputs.
 *   - One workspace must not be shared by calls that may run concurrently.
 *
 * Layouts (row-major, innermost last; B batch, H heads, n length, d head
 * dim, nb buckets, Rn rounds):
 *   x, v, out    [B][H][n][d]          in desc.dtype
 *   R            [Rn][d][nb/2]         in desc.dtype
 *   buckets      [B][H][Rn][n]         int32, position order
 *   perm         [B][H][Rn][n]         int32: perm[s] = position at sorted slot s
 *   xs, vs       [B][H][Rn][n][d]      desc.dtype, rows in sorted order
 *   lse          [B][H][Rn][n]         fp32, position order, natural log
 *
 * Supported (else LSH_ERR_UNSUPPORTED): dtype LSH_F32 or LSH_BF16; d in
 * {64, 128}; n_buckets even with 2 <= n_buckets <= 4096; chunk m >= 1 with
 * min(m, n) <= 128 and n % min(m, n) == 0 (m >= n is a single chunk);
 * 1 <= rounds <= 16; n * n_buckets < 2^31.
 */
#ifndef LSH_ATTN_H
#define LSH_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LSH_OK = 0,
    LSH_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum */
    LSH_ERR_UNSUPPORTED = 2, /* a valid problem outside the supported set */
    LSH_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
    LSH_ERR_CUDA = 4,        /* a CUDA runtime call failed */
    LSH_ERR_TIMEOUT = 5,     /* a kernel's bounded wait gave up */
    LSH_ERR_DEVICE = 6       /* a kernel rejected its input (bucket id range) */
} lsh_status;

typedef enum { LSH_F32 = 0, LSH_BF16 = 1 } lsh_dtype;

/* Problem description shared by every call. */
typedef struct {
    int32_t batch;     /* B >= 1 */
    int32_t heads;     /* H >= 1 */
    int32_t n;         /* sequence length >= 1 */
    int32_t d;         /* head dimension */
    int32_t n_buckets; /* nb: even, buckets per round */
    int32_t chunk;     /* m: chunk length in the sorted order */
    int32_t rounds;    /* independent hash rounds */
    int32_t causal;    /* 0 or 1 */
    int32_t dtype;     /* lsh_dtype of x, v, R, out, xs, vs */
} lsh_attn_desc;

/* Counters written by the kernels into the workspace header; reset at the
 * start of every hash / sort / forward call. */
typedef struct {
    uint32_t status;         /* lsh_status recorded by a kernel, 0 if none */
    uint32_t hash_refined;   /* (token, round) hashes re-decided in fp64 */
    uint32_t bad_bucket_ids; /* caller bucket ids outside [0, nb), clamped */
    uint32_t reserved;
} lsh_attn_diag;

/* Workspace bytes that lsh_attn_hash / lsh_attn_sort / lsh_attn_forward need
 * for `desc`. Writes *bytes; errors as for the calls themselves. */
lsh_status lsh_attn_workspace_size(const lsh_attn_desc *desc, size_t *bytes);

/* Hash every token in every round ("Reformer summary", §局部敏感哈希 and
 * §多輪LSH哈希): buckets[b][h][r][i] = argmax([x_i R_r ; -x_i R_r]), first
 * index on ties, bit-exact to the fp64 definition (bf16 runs on tensor cores
 * and re-decides near ties in fp64; fp32 runs in fp64).
 * x [B][H][n][d], R [Rn][d][nb/2] in desc.dtype; buckets out, int32. */
lsh_status lsh_attn_hash(const lsh_attn_desc *desc, const void *x, const void *R,
                         int32_t *buckets, void *workspace, size_t workspace_bytes,
                         void *stream);

/* Stable sort of every (batch, head, round) by bucket, then position
 * ("Reformer summary", §局部敏感哈希注意力): perm[s] = the position at sorted
 * slot s. If x, v, xs and vs are all non-NULL the rows of x and v are also
 * gathered into sorted order: xs[..][s] = x[..][perm[s]]; pass all four NULL
 * to skip the gather. buckets [B][H][Rn][n] int32 in [0, nb) (ids outside are
 * clamped and counted in the diag). */
lsh_status lsh_attn_sort(const lsh_attn_desc *desc, const int32_t *buckets, const void *x,
                         const void *v, int32_t *perm, void *xs, void *vs, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Whole forward pass: hash (skipped when `buckets` is non-NULL: the caller's
 * ids are used as given), sort and gather, chunked attention with unit keys,
 * 1/sqrt(d) scale, optional causal mask and the -1e5 self logit, un-sort, and
 * the logsumexp round merge. out [B][H][n][d] in desc.dtype; lse [B][H][Rn][n]
 * fp32 holds every round's log-normaliser in position order. */
lsh_status lsh_attn_forward(const lsh_attn_desc *desc, const void *x, const void *v,
                            const void *R, const int32_t *buckets, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Number of events lsh_attn_forward_profiled records. */
#define LSH_ATTN_PROFILE_EVENTS 10

/* lsh_attn_forward that also records the caller's CUDA events on `stream`
 * at every kernel boundary, for timing each kernel on the device:
 *   [0] start               [1] after the rotation transpose of the hash
 *   [2] after the projection / argmax kernel  [3] after the fp64 re-decision
 *   [4] after the bucket histograms  [5] after their scan
 *   [6] after the stable ranks (perm/inv)  [7] after the row gather
 *   [8] after the chunked attention  [9] after the un-sort and round merge
 * A kernel that does not run for this problem (caller-supplied buckets, the
 * fp64 hash) leaves consecutive events with nothing between them.
 * `events` points to LSH_ATTN_PROFILE_EVENTS cudaEvent_t handles created by
 * the caller. */
lsh_status lsh_attn_forward_profiled(const lsh_attn_desc *desc, const void *x, const void *v,
                                     const void *R, const int32_t *buckets, void *out, float *lse,
                                     void *workspace, size_t workspace_bytes, void *stream,
                                     void *const *events);

/* Synchronise `stream` and return the status the kernels recorded in
 * `workspace` since the last call that used it (LSH_OK if none). */
lsh_status lsh_attn_get_device_status(const void *workspace, void *stream);

/* Synchronise `stream` and copy the workspace counters into *diag. */
lsh_status lsh_attn_get_diag(const void *workspace, void *stream, lsh_attn_diag *diag);

/* Self-test of the bounded waits every kernel uses: clears the workspace
 * status word, then launches one CTA that waits on an mbarrier nothing
 * arrives at, with a limit of `limit_us` microseconds (1 .. 2000000) instead
 * of the kernels' 2 s. The wait gives up, the kernel records LSH_ERR_TIMEOUT
 * in the status word and returns, and the stream stays usable: read the
 * status with lsh_attn_get_device_status. `workspace` needs at least 256
 * bytes. Returns LSH_ERR_INVALID_ARG for a null workspace, too small a size
 * or a limit out of range (nothing is launched then). */
lsh_status lsh_attn_selftest_wait_timeout(void *workspace, size_t workspace_bytes,
                                          uint32_t limit_us, void *stream);

/* Size of the device-resident scratch of lsh_attn_sort_noalloc (8 MiB). */
#define LSH_ATTN_NOALLOC_SCRATCH_BYTES (8u << 20)

/* The stable sort of lsh_attn_sort (perm only, no row gather) for callers
 * that must not allocate device memory and cannot pass a workspace: for
 * example a plug-in whose host runtime owns all device memory, or a loop that
 * cannot afford the device synchronisation of cudaMalloc / cudaFree. The
 * paper has no counterpart to this entry point; it only changes where the
 * scratch lives. No memory is allocated: the scratch is a fixed array of
 * LSH_ATTN_NOALLOC_SCRATCH_BYTES in the library's own device memory, held by
 * every GPU that loads the library until the process exits.
 *   - buckets [B][H][Rn][n] int32 in; perm [B][H][Rn][n] int32 out (device).
 *   - A problem needs 256 + 4*B*H*Rn*nb*ceil(n / T) (rounded up to 256) +
 *     4*B*H*Rn*n bytes of scratch, T = 256 * clamp(8192 / nb, 1, 8); larger
 *     problems return LSH_ERR_UNSUPPORTED and write nothing (use lsh_attn_sort).
 *   - The first call on a device looks up the scratch's device address (with
 *     that device current) and caches it for the life of the process; make
 *     that first call before any stream capture. cudaDeviceReset on a device
 *     makes the cached address stale: after a reset, do not call this entry
 *     point on that device again in the same process.
 *   - Every call on a device shares the one scratch, whose contents persist
 *     from the previous call: calls that may overlap on the GPU (different
 *     streams without ordering between them) race and must not be issued.
 *   - Host-side errors as for lsh_attn_sort. The kernels' status word lives
 *     in the shared scratch and no call reads it, so bucket ids outside
 *     [0, nb) are clamped into range SILENTLY here (the perm is that of the
 *     clamped ids and the call returns LSH_OK); lsh_attn_sort reports the
 *     same input as LSH_ERR_DEVICE. */
lsh_status lsh_attn_sort_noalloc(const lsh_attn_desc *desc, const int32_t *buckets,
                                 int32_t *perm, void *stream);

/* Workspace bytes lsh_attn_dense_forward needs for `desc` (only batch,
 * heads, n, d, causal and dtype are read). Writes *bytes. */
lsh_status lsh_attn_dense_workspace_size(const lsh_attn_desc *desc, size_t *bytes);

/* Dense shared-QK attention, the full-attention baseline the pages compare
 * LSH attention with ("Reformer: LSH attention and reversible layers",
 * §三.3): every query attends to every key (causal: every key at an earlier
 * position) under the same rules as lsh_attn_forward's chunks -- keys scaled
 * to unit length, logits scaled by 1/sqrt(d), the -1e5 self logit -- so it
 * equals lsh_attn_forward with one round and one chunk spanning the sequence.
 *   x, v, out [B][H][n][d] bf16 (LSH_BF16 only, else LSH_ERR_UNSUPPORTED);
 *   lse [B][H][n] fp32, natural log. Any n >= 1; d in {64, 128};
 *   B * H * roundup(n, 128) < 2^31. n_buckets, chunk and rounds are ignored.
 *   workspace: lsh_attn_dense_workspace_size bytes, 256-byte aligned.
 * Conventions (ownership, asynchrony, errors) as for lsh_attn_forward. */
lsh_status lsh_attn_dense_forward(const lsh_attn_desc *desc, const void *x, const void *v,
                                  void *out, float *lse, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* Workspace bytes lsh_attn_backward needs for `desc`. Writes *bytes. */
lsh_status lsh_attn_backward_workspace_size(const lsh_attn_desc *desc, size_t *bytes);

/* Gradients of lsh_attn_forward with respect to x and v, for training
 * ("Reformer re-reading", §2.2, trains the model end to end). Bucket ids are
 * an input, as in the forward they were computed from (the hash is piecewise
 * constant and is not differentiated), and the sort is recomputed from them.
 *   x, v [B][H][n][d]; buckets [B][H][Rn][n]; out [B][H][n][d] and lse
 *   [B][H][Rn][n] from the forward on those inputs; dout = dL/dout
 *   [B][H][n][d]; dlse = dL/dlse [B][H][Rn][n] fp32 or NULL (zero);
 *   dx, dv [B][H][n][d] out. x, v, out, dout, dx, dv in desc.dtype.
 * Supported: LSH_BF16 with chunk 64 and n % 64 == 0 (else
 * LSH_ERR_UNSUPPORTED); other limits as for lsh_attn_forward.
 * The gradient is that of the definition: the self logit and masked keys
 * carry none, and the rounds' merge weights are differentiated; the round
 * outputs themselves are not needed (their term cancels). Deterministic.
 * Conventions (ownership, asynchrony, errors) as for lsh_attn_forward;
 * bucket ids outside [0, nb) are clamped and reported as there. */
lsh_status lsh_attn_backward(const lsh_attn_desc *desc, const void *x, const void *v,
                             const int32_t *buckets, const void *out, const float *lse,
                             const void *dout, const float *dlse, void *dx, void *dv,
                             void *workspace, size_t workspace_bytes, void *stream);

/* A reversible layer around the attention ("Reformer: LSH attention and
 * reversible layers", §二.2 reversible residual and §二.3 chunked
 * feed-forward): with x = [x1, x2],
 *   y1 = x1 + Attn(x2),   y2 = x2 + FFN(y1),
 * and back:  x2 = y2 - FFN(y1),   x1 = y1 - Attn(x2).
 * Attn(x) = W_o applied to the heads of lsh_attn_forward(x W_qk^T, x W_v^T)
 * (shared QK, d_model = heads * d_head), FFN(y) = max(y W1^T + b1, 0) W2^T
 * + b2 computed ffn_chunk rows at a time (the rows are independent, so the
 * chunk only bounds the intermediate buffer). */
typedef struct {
    int32_t batch, n;        /* sequences and their length (n % 128 == 0) */
    int32_t d_model;         /* = heads * d_head, a multiple of 128 */
    int32_t heads, d_head;   /* d_head in {64, 128} */
    int32_t d_ff;            /* feed-forward width, a multiple of 128 */
    int32_t ffn_chunk;       /* rows per feed-forward chunk, a multiple of 128 */
    int32_t n_buckets, chunk, rounds, causal;  /* the attention's (chunk 64) */
    int32_t hash_buckets;    /* forward: 1 = hash into `buckets`, 0 = read them */
} lsh_rev_desc;

/* Weights, bf16 stored out x in (row j holds output feature j), biases fp32
 * (either may be NULL for zero). */
typedef struct {
    const void *w_qk, *w_v, *w_o;  /* [d_model][d_model] */
    const void *w1;                /* [d_ff][d_model] */
    const float *b1;               /* [d_ff] */
    const void *w2;                /* [d_model][d_ff] */
    const float *b2;               /* [d_model] */
} lsh_rev_weights;

/* Workspace bytes lsh_rev_block needs for `desc`. */
lsh_status lsh_rev_workspace_size(const lsh_rev_desc *desc, size_t *bytes);

/* inverse = 0: (in1, in2) = (x1, x2) -> (out1, out2) = (y1, y2); the bucket
 * ids [batch][heads][rounds][n] are hashed from x2 W_qk^T under R into
 * `buckets` (desc.hash_buckets = 1) or read from it (0).
 * inverse = 1: (in1, in2) = (y1, y2) -> (out1, out2) = (x1, x2) with the
 * forward's bucket ids read from `buckets` (R unused).
 * All activations [batch][n][d_model] bf16, device memory, 16-byte aligned.
 * Kernel status (the products' and the attention's) is read with
 * lsh_attn_get_device_status(workspace). Other conventions as for
 * lsh_attn_forward. */
lsh_status lsh_rev_block(const lsh_rev_desc *desc, int inverse, const void *in1, const void *in2,
                         const lsh_rev_weights *weights, const void *R, int32_t *buckets,
                         void *out1, void *out2, void *workspace, size_t workspace_bytes,
                         void *stream);

/* The in-bucket top-k variant of LSH attention ("Reformer re-reading",
 * §2.2), a second workload beside lsh_attn_forward: per round l, bucket(x) =
 * (sum_t [proj_l[:, t] . x > 0] 2^t) mod n_buckets over n_bits projections;
 * every query ranks the keys of its bucket (causal: positions <= its own) by
 * the chunked attention's logit x_i . x_j / (||x_j|| sqrt(d)) (-1e5 for
 * itself; higher first, lower position on ties) and keeps the top_k; the
 * candidates are the union over rounds, attended with one softmax of those
 * logits. Bucket bits and top-k sets are decided in fp64 (sums in increasing
 * feature order, no fused multiply-add); the softmax runs in fp32. */
typedef struct {
    int32_t batch, heads, n, d;  /* d in {64, 128} */
    int32_t n_buckets;           /* K: even, 2 .. 4096 */
    int32_t n_bits;              /* m projections per round, 1 .. 32 */
    int32_t top_k;               /* 1 .. 32 */
    int32_t rounds;              /* L: 1 .. 8 */
    int32_t causal;
} lsh_topk_desc;

/* Workspace bytes lsh_topk_forward needs for `desc`. */
lsh_status lsh_topk_workspace_size(const lsh_topk_desc *desc, size_t *bytes);

/* x, v, out [B][H][n][d] bf16; proj [rounds][d][n_bits] bf16; lse [B][H][n]
 * fp32; cand (optional, else kept in the workspace) [B][H][rounds][n][top_k]
 * int32: each round's top-k positions, best first, -1 past the kept ones.
 * Conventions as for lsh_attn_forward. */
lsh_status lsh_topk_forward(const lsh_topk_desc *desc, const void *x, const void *v,
                            const void *proj, void *out, float *lse, int32_t *cand,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Static, human-readable name of a status code. */
const char *lsh_attn_status_string(lsh_status status);

#ifdef __cplusplus
}
#endif

#endif /* LSH_ATTN_H */
