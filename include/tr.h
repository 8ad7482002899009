/*
 * tr.h -- C ABI of the TransRetrieval candidate-scoring library (libtr.so).
 *
 * The four calls of the scoring path, from "TransRetrieval: Scaling Up Transformer-Based
 * Retrieval for Industrial Recommendation":
 *   tr_aggregate         weighted-average aggregation of (key, weight) fields      (§3.2)
 *   tr_prefill_user      user tokens + domain embedding through the N-layer Pre-LN
 *                        Transformer, writing the per-layer user K/V cache          (§3.1, §3.4)
 *   tr_compress_targets  3-layer MLP target compressor, F*D -> D                    (§3.3)
 *   tr_compress_target_bags  the aggregation of the target fields feeding the compressor
 *                        in one launch, the compressor's input built on chip (§3.2 + §3.3)
 *   tr_score_candidates  single-token candidates through the same layer stack over
 *                        the broadcast user K/V, then the linear head; candidates of
 *                        several requests packed in one call, each isolated to its
 *                        own request                       (§3.3, deployment section)
 *
 * Conventions
 *  - Every call returns tr_status.  TR_OK is 0.  On failure, tr_last_error() returns a
 *    thread-local message describing the first problem found.
 *  - Arguments are validated on the host before anything is launched; an invalid call
 *    launches nothing and writes nothing.
 *  - Compute calls are asynchronous on the caller's CUDA stream (tr_stream is a
 *    cudaStream_t; NULL means the legacy default stream).  Errors that only the device
 *    can see (a key outside its table) do not stop the kernel: the offending key is
 *    skipped and a device status word is set; tr_sync_status() reports it.
 *  - The caller owns every input/output device buffer.  The library owns the model
 *    handle (its repacked weights, released by tr_model_destroy()), a status word per
 *    device, and scratch for the calls that run as a sequence of CUDA-core kernels (fp32
 *    models, user sides or score calls with more than 128 user tokens, the uncompressed-
 *    target variant): one buffer per (device, stream), kept until process exit.  Calls on
 *    different streams never share scratch; calls on one stream are ordered by it.  A call
 *    that needs more scratch than its stream's buffer holds synchronises that stream and
 *    reallocates it, so the first such call on a stream must not be made while the stream
 *    is being captured into a CUDA graph.  The tensor-core paths use no scratch; the
 *    tensor-core compressor of a TR_BF16 model takes its tiles from a work counter, a few
 *    device ints per (device, stream) that the library allocates (zeroed) on the first
 *    such call on a stream, kept until process exit, and zeroes on the stream before every
 *    launch; the same capture rule applies to that first call.
 *  - Row-major layouts unless stated; "[a][b]" means a rows of b contiguous elements.
 *  - dtype TR_F32 models compute in fp32 throughout.  TR_BF16 models store tables,
 *    weights and target-field tokens in bf16; the compressed candidate tokens are fp32 for
 *    every model.  The tensor-core kernels of a TR_BF16 model multiply fp16 operands (the
 *    bf16 weights converted exactly, activations rounded to fp16's 11-bit significand),
 *    except the compressor's first layer, which multiplies the bf16 field tokens by bf16
 *    weights; every product accumulates in fp32.  A TR_BF16 model whose LayerNorm gains
 *    and weights could push an fp16 operand out of range runs on the CUDA-core kernels.
 */
#ifndef TR_H
#define TR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int tr_status;
#define TR_OK 0
#define TR_ERR_INVALID_ARG 1  /* bad pointer, size, dtype or index; nothing launched        */
#define TR_ERR_UNSUPPORTED 2  /* valid but not implemented (e.g. a model size)              */
#define TR_ERR_CUDA 3         /* a CUDA runtime call failed; message has the CUDA error      */
#define TR_ERR_KEY_RANGE 4    /* device saw a key >= its table's rows (that key was skipped) */
#define TR_ERR_TIMEOUT 5      /* tr_sync_status() deadline passed before the stream drained */
#define TR_ERR_NOMEM 6        /* device allocation for the model or workspace failed         */

typedef enum { TR_F32 = 0, TR_BF16 = 1 } tr_dtype;

typedef void* tr_stream; /* cudaStream_t */

#define TR_MAX_TABLES 64     /* tables per tr_aggregate call            */
#define TR_MAX_REQUESTS 64   /* requests packed in one score call      */
#define TR_MAX_LU 256        /* user tokens per request                */

/* Model sizes (TransRetrieval §4.1 xD-yL notation). */
typedef struct {
  int D;               /* token width; multiple of 16, <= 128                        */
  int n_layer;         /* Transformer layers, 1..16                                  */
  int n_head;          /* heads; d_h = D / n_head must be 16                         */
  int ffn_hidden;      /* FFN hidden width (2*D for the paper's FLOP count)          */
  int n_target_fields; /* F                                                          */
  int comp_dims[4];    /* compressor F*D -> c1 -> c2 -> D; comp_dims[0] == F*D,
                          comp_dims[3] == D                                          */
  int n_domains;       /* domain embeddings s_d                                      */
  tr_dtype dtype;
} tr_model_desc;

/* One layer's parameters: HOST pointers to fp32 arrays.  Linear maps are W[in][out]
 * with y = x W + b.  For TR_BF16 models every value must be exactly representable in
 * bf16 (it is converted without rounding checks). */
typedef struct {
  const float *ln1_g, *ln1_b;             /* [D]                         */
  const float *Wq, *bq, *Wk, *bk, *Wv, *bv; /* [D][D], [D]                 */
  const float *Wo, *bo;                   /* [D][D], [D]                  */
  const float *ln2_g, *ln2_b;             /* [D]                          */
  const float *W1, *b1;                   /* [D][ffn_hidden], [ffn_hidden] */
  const float *W2, *b2;                   /* [ffn_hidden][D], [D]         */
} tr_layer_weights;

typedef struct {
  const float* domain_emb;          /* [n_domains][D]                                */
  const tr_layer_weights* layers;   /* host array [n_layer]                          */
  const float *lnf_g, *lnf_b;       /* [D] final LayerNorm                           */
  const float* w_head;              /* [D]                                           */
  float b_head;
  const float* comp_W[3];           /* [comp_dims[i]][comp_dims[i+1]]                */
  const float* comp_b[3];           /* [comp_dims[i+1]]                              */
  const float* comp_prelu[2];       /* [comp_dims[i+1]] PReLU slopes                 */
  const float* comp_ln_g[2];        /* [comp_dims[i+1]]                              */
  const float* comp_ln_b[2];
} tr_model_weights;

typedef struct tr_model tr_model;

/* Embedding table: DEVICE pointer to [n_rows][D] values of type dtype. */
typedef struct {
  const void* data;
  int64_t n_rows;
  tr_dtype dtype;
} tr_table;

const char* tr_last_error(void);

/* Copies and repacks the weights into device memory owned by the returned handle.
 * Uses the current CUDA device.  Synchronous.  With the environment variable
 * TR_FORCE_SIMT=1 at creation time, a bf16 model runs every stage on the CUDA-core
 * (fp32 arithmetic) kernels instead of the tensor-core ones. */
tr_status tr_model_create(const tr_model_desc* desc, const tr_model_weights* w, tr_model** out);
void tr_model_destroy(tr_model* m);

/*
 * Weighted-average aggregation (TransRetrieval §3.2): for every bag b
 *     out[b] = sum_{i in bag b} weights[i] * table[bag_table[b]][keys[i]] / sum_{i in b} weights[i]
 * accumulated in fp32; the division is a multiplication by the correctly rounded fp32
 * reciprocal of the weight sum, so scaling every weight of a bag by a power of two leaves
 * the result bit-identical.  A bag with no keys, or whose weights sum to exactly 0, yields
 * the zero vector.  Duplicate keys count once per occurrence.
 *   tables     HOST array [n_tables] (<= TR_MAX_TABLES); all tables share one dtype
 *   bag_table  DEVICE int32 [n_bags], each in [0, n_tables)  (validated on the device:
 *              an out-of-range entry zeroes the bag and sets TR_ERR_KEY_RANGE)
 *   offsets    DEVICE int64 [n_bags + 1], non-decreasing, offsets[0] = 0
 *   keys       DEVICE int32 [offsets[n_bags]]; a key >= n_rows (or < 0) is skipped and
 *              sets the device status word (TR_ERR_KEY_RANGE via tr_sync_status)
 *   weights    DEVICE fp32  [offsets[n_bags]]
 *   out        DEVICE [n_bags][D] of out_dtype.  For the compressor input, bag
 *              b = c*F + f gives out viewed as [n_cand][F*D].
 * D must be a multiple of 8 and <= 512.  n_bags = 0 is a no-op.
 */
tr_status tr_aggregate(const tr_table* tables, int n_tables, const int32_t* bag_table,
                       const int64_t* offsets, const int32_t* keys, const float* weights,
                       int64_t n_bags, int D, tr_dtype out_dtype, void* out, tr_stream stream);

/*
 * Aggregator variants of tr_aggregate (TransRetrieval §3.2 names them as the alternatives
 * weighted average replaces; they are here for that comparison).  Same arguments and layout
 * as tr_aggregate plus `mode`:
 *   TR_AGG_MEAN  sum_i v_i h(k_i) / sum_i v_i   (tr_aggregate; zero when sum_i v_i = 0)
 *   TR_AGG_SUM   sum_i v_i h(k_i)               (the weighted sum of §3.2's profiling paragraph)
 *   TR_AGG_MAX   max_i h(k_i) element-wise     (max pooling; weights unused; empty bag -> 0)
 * optionally OR-ed with
 *   TR_AGG_POST_LN  LayerNorm over the D columns of each token, without gain or shift, eps 1e-5
 *                   (post-aggregation LayerNorm).
 * Any other value is rejected with TR_ERR_INVALID_ARG.
 */
#define TR_AGG_MEAN 0
#define TR_AGG_SUM 1
#define TR_AGG_MAX 2
#define TR_AGG_POST_LN 0x100
tr_status tr_aggregate_ex(const tr_table* tables, int n_tables, const int32_t* bag_table, const int64_t* offsets,
                          const int32_t* keys, const float* weights, int64_t n_bags, int D, tr_dtype out_dtype,
                          int mode, void* out, tr_stream stream);

/*
 * Bytes of one request's user K/V cache for L_u user tokens (0 <= L_u <= TR_MAX_LU).
 * Layout (opaque to most callers; tests decode it):
 *   TR_F32 model : [n_layer][2][L_u][D] fp32, K then V, row-major.
 *   TR_BF16 model: per layer a K image then a V image, fp16, in the tensor-core operand
 *   layout.  With Lp = L_u rounded up to 16 (rows >= L_u are zero) and 8x8 "core
 *   matrices" of 128 contiguous bytes (8 rows of 8 consecutive elements):
 *     K image  [Lp x D]: element (j, d) at core (d/8)*(Lp/8) + j/8, within it (j%8)*8 + d%8
 *     V image  [D x Lp] (V transposed): element (d, j) at core (j/8)*(D/8) + d/8,
 *              within it (d%8)*8 + j%8
 *   each image is Lp*D*2 bytes; layer l starts at l * 2*Lp*D*2 bytes.
 */
size_t tr_kv_cache_bytes(const tr_model* m, int L_u);

/*
 * User side of one request (TransRetrieval §3.1 stages (3)-(4), §3.4): x = user_tokens
 * + s_domain, then for each layer a Pre-LN attention block (every user token attends to
 * every user token) and a Pre-LN ReLU FFN block; the layer's K = LN1(x) Wk + bk and
 * V = LN1(x) Wv + bv are written to kv (layout above).
 *   user_tokens DEVICE fp32 [L_u][D];  kv DEVICE buffer of tr_kv_cache_bytes(m, L_u).
 * L_u = 0 writes nothing.
 */
tr_status tr_prefill_user(const tr_model* m, const float* user_tokens, int L_u, int domain,
                          void* kv, tr_stream stream);

/*
 * The user sides of R requests in one call: tr_prefill_user for every request r, run as one
 * launch of one tensor-core CTA per request when the model and every L_u (<= 128) allow it,
 * else one call after the other.  Requests with L_u[r] = 0 write nothing.
 *   user_tokens HOST array [R] of DEVICE fp32 [L_u[r]][D]
 *   L_u, domain HOST int32 [R]
 *   kv          HOST array [R] of DEVICE buffers of tr_kv_cache_bytes(m, L_u[r]) bytes
 * 1 <= R <= TR_MAX_REQUESTS.  Every argument is validated before anything is launched.
 */
tr_status tr_prefill_users(const tr_model* m, const float* const* user_tokens, const int32_t* L_u,
                           const int32_t* domain, void* const* kv, int R, tr_stream stream);

/*
 * Target compressor (TransRetrieval §3.3): t = W3 g2(W2 g1(W1 x + b1) + b2) + b3 with
 * g_i(z) = LayerNorm_i(PReLU_i(z)).
 *   x      DEVICE [n][comp_dims[0]] of the model dtype (the concatenated field tokens)
 *   tokens DEVICE fp32 [n][D].
 */
tr_status tr_compress_targets(const tr_model* m, const void* x, int64_t n, void* tokens,
                              tr_stream stream);

/*
 * The target side in one launch: the weighted-average aggregation of TransRetrieval §3.2
 * feeding the compressor of §3.3, whose input row (the concatenation of a candidate's F
 * field tokens) is built in shared memory and never written to device memory.  Candidate c's
 * field f is bag c*F + f (F = n_target_fields), as tr_aggregate lays the rows of x out; its
 * token is rounded to bf16 exactly as tr_aggregate(..., TR_BF16, ...) rounds it, so the
 * result equals tr_aggregate followed by tr_compress_targets bit for bit, except where
 * tr_aggregate takes its few-bags path (at most 4 bags per SM), which sums in another order.
 *   tables     HOST array [n_tables] of bf16 tables of width D (DEVICE data, 16-byte aligned)
 *   bag_table  DEVICE int32 [n*F]      table of each bag (outside 0..n_tables-1: token 0)
 *   offsets    DEVICE int64 [n*F + 1]  CSR offsets into keys / weights
 *   keys       DEVICE int32, weights DEVICE fp32 (a key outside its table is skipped and
 *              sets the device status, as in tr_aggregate)
 *   tokens     DEVICE fp32 [n][D], 16-byte aligned.
 * Needs a TR_BF16 model served by the tensor-core compressor with D a multiple of 64 and
 * comp_dims[0] == F*D; otherwise TR_ERR_UNSUPPORTED and nothing is launched.  Uses the same
 * per-stream work counter as tr_compress_targets.
 */
tr_status tr_compress_target_bags(const tr_model* m, const tr_table* tables, int n_tables,
                                  const int32_t* bag_table, const int64_t* offsets,
                                  const int32_t* keys, const float* weights, int64_t n,
                                  void* tokens, tr_stream stream);

/*
 * Score packed candidates (TransRetrieval §3.3 and deployment "Hardware-aware inference
 * optimization").  Candidates of request r are rows req_offsets[r] .. req_offsets[r+1]-1;
 * each runs as one token y = t + s_domain[r] through every layer: Pre-LN multi-head
 * attention over its request's L_u cached user keys/values plus its own key/value,
 * then the Pre-LN ReLU FFN; score = w_head . LayerNorm_f(y) + b_head.  A candidate never
 * sees another candidate or another request's cache.
 *   tokens      DEVICE fp32 [n][D] (as tr_compress_targets writes them)
 *   req_offsets HOST int64 [R+1], req_offsets[0] = 0, non-decreasing, req_offsets[R] = n
 *   kv          HOST array [R] of DEVICE pointers (caches written by tr_prefill_user)
 *   L_u, domain HOST int32 [R]
 *   scores      DEVICE fp32 [n]
 * 1 <= R <= TR_MAX_REQUESTS.
 */
tr_status tr_score_candidates(const tr_model* m, const void* tokens, int64_t n,
                              const int64_t* req_offsets, const void* const* kv,
                              const int32_t* L_u, const int32_t* domain, int R, float* scores,
                              tr_stream stream);

/*
 * The uncompressed-target variant (TransRetrieval §3.3 compares against it): each candidate
 * is L_t target tokens instead of one compressed token.  Every token runs through the same
 * layer stack, attending to its request's L_u cached user keys/values and to the keys/values
 * of its own candidate's L_t tokens (never another candidate's); the candidate's score is the
 * mean over its tokens of w_head . LayerNorm_f(y_t) + b_head.  With L_t = 1 this is
 * tr_score_candidates.  It exists to measure the per-candidate cost that target compression
 * removes.  A TR_BF16 model on the tensor-core stack with L_t a power of two up to 16 (and
 * every L_u <= 128) runs it in the same kernel as tr_score_candidates, a candidate's tokens
 * being L_t consecutive rows of a tile whose own-candidate attention runs on CUDA cores
 * (and with L_t = 1 its scores equal tr_score_candidates' on the same token values bit for
 * bit); any other case runs the CUDA-core kernels (fp32 arithmetic).
 *   tokens      DEVICE [n][L_t][D] of the model dtype (candidate c's tokens are rows c*L_t ..)
 *   L_t         1 .. TR_MAX_LT
 *   req_offsets, kv, L_u, domain, R, scores: as tr_score_candidates (n counts candidates).
 */
#define TR_MAX_LT 16
tr_status tr_score_candidates_uncompressed(const tr_model* m, const void* tokens, int64_t n, int L_t,
                                           const int64_t* req_offsets, const void* const* kv, const int32_t* L_u,
                                           const int32_t* domain, int R, float* scores, tr_stream stream);

/*
 * Per-request top-k of the scores (the selection step of GPU retrieval, TransRetrieval
 * deployment section "Hardware-aware inference optimization": a request's scored candidates
 * are reduced to the best k on the GPU).
 *   scores      DEVICE fp32 [n], candidates grouped by request as in tr_score_candidates
 *   req_offsets HOST int64 [R+1], req_offsets[0] = 0, non-decreasing, req_offsets[R] = n
 *   k           1 .. TR_MAX_TOPK
 *   out_idx     DEVICE int64 [R][k]: for request r, candidate indices within the request
 *               (0-based) by descending score; equal scores by lower index; a request with
 *               fewer than k candidates is padded with -1
 *   out_score   DEVICE fp32 [R][k] or NULL: the selected scores (padding -inf)
 * NaN scores rank below every other score.  The selected set and its order are unique, so
 * the result does not depend on the launch or on other requests.  1 <= R <= TR_MAX_REQUESTS.
 */
#define TR_MAX_TOPK 4096
tr_status tr_topk(const float* scores, int64_t n, const int64_t* req_offsets, int R, int k, int64_t* out_idx,
                  float* out_score, tr_stream stream);

/*
 * No-allocation variant of tr_prefill_user.  The paper has no counterpart: this entry point
 * exists for callers that cannot call cudaMalloc when the user side runs -- code running
 * while a CUDA stream capture is open (allocation is not a capturable operation), serving
 * engines whose own allocator owns all device memory, and latency-critical loops that cannot
 * afford the device-wide synchronisation a growing workspace costs.  tr_prefill_user itself
 * allocates nothing on the tensor-core path, but its CUDA-core path grows a library-owned
 * workspace with cudaMalloc.
 *
 * This call runs the CUDA-core (fp32 arithmetic) user side for any model dtype, with its
 * scratch in one file-scope device array of TR_NOALLOC_SCRATCH_BYTES that every GPU loading
 * the library holds until process exit.  It calls no cudaMalloc, cudaFree or allocating
 * library routine.  Arguments and output are those of tr_prefill_user; for a TR_BF16 model the
 * result agrees with tr_prefill_user within the bf16 tolerance, not bit for bit.
 *   Limit: L_u * (6*D + ffn_hidden) * 4 bytes <= TR_NOALLOC_SCRATCH_BYTES (with D = 128 and
 *          ffn_hidden = 256 that is every L_u <= TR_MAX_LU); a larger request is rejected with
 *          TR_ERR_INVALID_ARG before anything is launched.
 *   Sharing: every call on a device uses the same array, which keeps the last call's
 *          contents (nothing in it has to start at zero: each call writes every element it
 *          reads).  Calls whose kernels overlap on the GPU -- different streams, or several
 *          host threads -- race on the array; serialise them.
 *   Set-up: the first call on each device looks up the array's device address (and may load
 *          the library's device code) with that device current; make that first call before
 *          any stream capture begins.
 */
#define TR_NOALLOC_SCRATCH_BYTES (1u << 20)
tr_status tr_prefill_user_noalloc(const tr_model* m, const float* user_tokens, int L_u, int domain,
                                  void* kv, tr_stream stream);

/*
 * Waits for `stream` (polling, up to timeout_ms; <= 0 means no limit), then reads and
 * clears this device's status word.  Returns TR_ERR_TIMEOUT if the stream did not drain
 * in time (the status word is left untouched), TR_ERR_KEY_RANGE if a kernel reported an
 * out-of-range key or table index since the last call, else TR_OK.
 */
tr_status tr_sync_status(tr_stream stream, int timeout_ms);

/* Library version, for diagnostics. */
const char* tr_version(void);

/* Number of kernels this library has launched in this process (all devices, all
 * threads); a diagnostic for counting launches inside a timed region. */
unsigned long long tr_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* TR_H */
