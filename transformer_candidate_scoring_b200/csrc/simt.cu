// fp32 CUDA-core path of every stage except aggregation.
//
// This is the arithmetic of TR_F32 models (the 1e-4 parity tier, which neither bf16 nor
// TF32 operands can meet) and the fallback for shapes the tensor-core kernels do not
// take.  Stages run as a short sequence of plain kernels over an fp32 workspace:
// tiled GEMM with fused bias / ReLU / residual, row LayerNorm (optionally after PReLU),
// one-warp-per-(row, head) attention.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "model.cuh"

namespace tr {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;
enum { EPI_NONE = 0, EPI_RELU = 1, EPI_ACCUM = 2 };

// C[m][n] (=|+=) act(sum_k A[m][k] B[k][n] + bias[n])
template <typename TA>
__global__ void __launch_bounds__(256) gemm_kernel(const TA* __restrict__ A, int lda, const float* __restrict__ B,
                                                   int ldb, const float* __restrict__ bias, float* __restrict__ C,
                                                   int ldc, int M, int N, int K, int epi) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int gm = m0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? to_f32(A[(int64_t)gm * lda + gk]) : 0.f;
    }
    for (int i = threadIdx.x; i < BK * BN; i += 256) {
      const int r = i / BN, c = i % BN;
      const int gk = k0 + r, gn = n0 + c;
      Bs[r][c] = (gk < K && gn < N) ? B[(int64_t)gk * ldb + gn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= N) continue;
      float v = acc[i][j] + (bias ? bias[gn] : 0.f);
      if (epi & EPI_RELU) v = fmaxf(v, 0.f);
      float* c = C + (int64_t)gm * ldc + gn;
      *c = (epi & EPI_ACCUM) ? *c + v : v;
    }
  }
}

template <typename TA>
tr_status gemm(const TA* A, int lda, const float* B, int ldb, const float* bias, float* C, int ldc, int M, int N,
               int K, int epi, cudaStream_t st) {
  if (M == 0) return TR_OK;
  dim3 grid(ceil_div(N, BN), ceil_div(M, BM));
  gemm_kernel<TA><<<grid, 256, 0, st>>>(A, lda, B, ldb, bias, C, ldc, M, N, K, epi);
  TR_LAUNCH_CHECK("gemm_kernel");
  return TR_OK;
}

// Y = LayerNorm(prelu ? PReLU(X) : X) * g + b over rows of width N; one warp per row.
template <typename TY>
__global__ void layernorm_rows(const float* __restrict__ X, int ldx, TY* __restrict__ Y, int ldy, int M, int N,
                               const float* __restrict__ prelu, const float* __restrict__ g,
                               const float* __restrict__ b) {
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* x = X + (int64_t)row * ldx;
  auto val = [&](int i) {
    float v = x[i];
    if (prelu && v < 0.f) v *= prelu[i];
    return v;
  };
  float s = 0.f;
  for (int i = lane; i < N; i += 32) s += val(i);
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mu = s / N;
  float q = 0.f;
  for (int i = lane; i < N; i += 32) {
    const float d = val(i) - mu;
    q += d * d;
  }
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / N + kLnEps);
  TY* y = Y + (int64_t)row * ldy;
  for (int i = lane; i < N; i += 32) y[i] = from_f32<TY>((val(i) - mu) * rstd * g[i] + b[i]);
}

template <typename TY>
tr_status layernorm(const float* X, int ldx, TY* Y, int ldy, int M, int N, const float* prelu, const float* g,
                    const float* b, cudaStream_t st) {
  if (M == 0) return TR_OK;
  layernorm_rows<TY><<<ceil_div(M, 8), 256, 0, st>>>(X, ldx, Y, ldy, M, N, prelu, g, b);
  TR_LAUNCH_CHECK("layernorm_rows");
  return TR_OK;
}

// Y[m][d] = X[m][d] + s[d]
template <typename TX>
__global__ void add_vec_rows(const TX* __restrict__ X, float* __restrict__ Y, int64_t M, int D,
                             const float* __restrict__ s) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * D) return;
  Y[i] = to_f32(X[i]) + s[i % D];
}

// Cached user K/V of one layer, in either cache layout.
struct KvF32 {
  const float* K;  // [L_u][D]
  const float* V;
  int ld;
  __device__ float k(int j, int d) const { return K[(int64_t)j * ld + d]; }
  __device__ float v(int j, int d) const { return V[(int64_t)j * ld + d]; }
};
struct KvF16Image {
  const __half* K;  // [Lp x D] core-matrix image
  const __half* V;  // [D x Lp] core-matrix image
  int Lp, D;
  __device__ float k(int j, int d) const {
    return __half2float(K[((d >> 3) * (Lp >> 3) + (j >> 3)) * 64 + (j & 7) * 8 + (d & 7)]);
  }
  __device__ float v(int j, int d) const {
    return __half2float(V[((j >> 3) * (D >> 3) + (d >> 3)) * 64 + (d & 7) * 8 + (j & 7)]);
  }
};

// One warp per (row, head): softmax over the L_u user keys plus the keys of the row's own
// candidate (Lt rows: rows (row / Lt) * Lt .. + Lt - 1, i.e. the row itself when Lt = 1,
// none when Lt = 0) of q.k / sqrt(d_h), then the weighted sum of values.
constexpr int kMaxLt = 16;
template <typename KV>
__global__ void attention_rows(const float* __restrict__ q, int ldq, const float* __restrict__ kself,
                               const float* __restrict__ vself, int ldself, KV kv, int L_u, int M, int H,
                               float* __restrict__ o, int ldo, int Lt) {
  const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)M * H) return;
  const int row = (int)(w / H), h = (int)(w % H);
  const float scale = 0.25f;  // 1/sqrt(16)
  float qv[kDHead];
#pragma unroll
  for (int d = 0; d < kDHead; ++d) qv[d] = q[(int64_t)row * ldq + h * kDHead + d];
  constexpr int MAXT = TR_MAX_LU / 32;
  float s[MAXT];
  float mx = -INFINITY;
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    const int j = lane + 32 * t;
    s[t] = -INFINITY;
    if (j < L_u) {
      float a = 0.f;
#pragma unroll
      for (int d = 0; d < kDHead; ++d) a = fmaf(qv[d], kv.k(j, h * kDHead + d), a);
      s[t] = a * scale;
      mx = fmaxf(mx, s[t]);
    }
  }
  const int64_t g0 = Lt > 0 ? (int64_t)(row / Lt) * Lt : 0;   // first row of this candidate
  float sself[kMaxLt];
#pragma unroll
  for (int t = 0; t < kMaxLt; ++t) {
    sself[t] = -INFINITY;
    if (t < Lt) {
      float a = 0.f;
#pragma unroll
      for (int d = 0; d < kDHead; ++d) a = fmaf(qv[d], kself[(g0 + t) * ldself + h * kDHead + d], a);
      sself[t] = a * scale;
    }
  }
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
#pragma unroll
  for (int t = 0; t < kMaxLt; ++t) mx = fmaxf(mx, sself[t]);
  float acc[kDHead] = {};
  float sum = 0.f;
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    const int j = lane + 32 * t;
    if (j < L_u) {
      const float p = __expf(s[t] - mx);
      sum += p;
#pragma unroll
      for (int d = 0; d < kDHead; ++d) acc[d] = fmaf(p, kv.v(j, h * kDHead + d), acc[d]);
    }
  }
  for (int off = 16; off; off >>= 1) {
    sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
    for (int d = 0; d < kDHead; ++d) acc[d] += __shfl_xor_sync(0xffffffffu, acc[d], off);
  }
#pragma unroll
  for (int t = 0; t < kMaxLt; ++t) {
    if (t < Lt) {
      const float p = __expf(sself[t] - mx);
      sum += p;
#pragma unroll
      for (int d = 0; d < kDHead; ++d) acc[d] = fmaf(p, vself[(g0 + t) * ldself + h * kDHead + d], acc[d]);
    }
  }
  if (lane < kDHead) {
    float r = 0.f;
#pragma unroll
    for (int d = 0; d < kDHead; ++d)
      if (d == lane) r = acc[d];
    o[(int64_t)row * ldo + h * kDHead + lane] = r / sum;
  }
}

// Writes layer l's K and V (columns D..2D-1 and 2D..3D-1 of qkv) into the cache.
__global__ void kv_write_f32(const float* __restrict__ qkv, int L_u, int D, float* __restrict__ cache_l) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * L_u * D) return;
  const int which = i / (L_u * D), r = i % (L_u * D);
  const int j = r / D, d = r % D;
  cache_l[i] = qkv[(int64_t)j * 3 * D + (1 + which) * D + d];
}

__global__ void kv_write_f16(const float* __restrict__ qkv, int L_u, int Lp, int D, __half* __restrict__ cache_l) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= 2 * Lp * D) return;
  const bool isv = i >= Lp * D;
  const int r = isv ? i - Lp * D : i;
  const int core = r >> 6, within = r & 63;
  int j, d;
  if (!isv) {  // K image: core = (d/8)*(Lp/8) + j/8, within = (j%8)*8 + d%8
    d = (core / (Lp >> 3)) * 8 + (within & 7);
    j = (core % (Lp >> 3)) * 8 + (within >> 3);
  } else {     // V image: core = (j/8)*(D/8) + d/8, within = (d%8)*8 + j%8
    j = (core / (D >> 3)) * 8 + (within & 7);
    d = (core % (D >> 3)) * 8 + (within >> 3);
  }
  const float v = (j < L_u) ? qkv[(int64_t)j * 3 * D + (isv ? 2 : 1) * D + d] : 0.f;
  cache_l[i] = __float2half_rn(v);
}

// score = w . LayerNorm_f(y) + b; one warp per row.
__global__ void head_rows(const float* __restrict__ Y, int64_t M, int D, const float* __restrict__ g,
                          const float* __restrict__ b, const float* __restrict__ w, float bh,
                          float* __restrict__ out) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const float* y = Y + row * D;
  float s = 0.f;
  for (int i = lane; i < D; i += 32) s += y[i];
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mu = s / D;
  float q = 0.f;
  for (int i = lane; i < D; i += 32) q += (y[i] - mu) * (y[i] - mu);
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / D + kLnEps);
  float acc = 0.f;
  for (int i = lane; i < D; i += 32) acc += ((y[i] - mu) * rstd * g[i] + b[i]) * w[i];
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[row] = acc + bh;
}

template <typename TO>
__global__ void convert_rows(const float* __restrict__ X, TO* __restrict__ Y, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) Y[i] = from_f32<TO>(X[i]);
}

// One Pre-LN layer over M rows held in y (fp32 [M][D]); attention reads `kv`.
template <typename KV>
tr_status layer(const tr_model* m, int l, float* y, float* a, float* qkv, float* o, float* hbuf, int M, KV kv,
                int L_u, int lt, void* kv_out, cudaStream_t st) {
  const int D = m->desc.D, H = m->desc.ffn_hidden, NH = m->desc.n_head;
  const tr_layer_dev& L = m->layers[l];
  TR_TRY(layernorm<float>(y, D, a, D, M, D, nullptr, L.ln1_g, L.ln1_b, st));
  TR_TRY(gemm<float>(a, D, L.Wqkv, 3 * D, L.bqkv, qkv, 3 * D, M, 3 * D, D, EPI_NONE, st));
  if (kv_out) {  // prefill: this layer's K/V are the users' own
    if (m->desc.dtype == TR_F32) {
      kv_write_f32<<<ceil_div(2 * M * D, 256), 256, 0, st>>>(qkv, M, D, (float*)kv_out);
    } else {
      const int Lp = round_up16(M);
      kv_write_f16<<<ceil_div(2 * Lp * D, 256), 256, 0, st>>>(qkv, M, Lp, D, (__half*)kv_out);
    }
    TR_LAUNCH_CHECK("kv_write");
  }
  const int64_t warps = (int64_t)M * NH;
  attention_rows<KV><<<ceil_div(warps, 8), 256, 0, st>>>(qkv, 3 * D, qkv + D, qkv + 2 * D, 3 * D, kv, L_u, M, NH, o,
                                                          D, lt);
  TR_LAUNCH_CHECK("attention_rows");
  TR_TRY(gemm<float>(o, D, L.Wo, D, L.bo, y, D, M, D, D, EPI_ACCUM, st));
  TR_TRY(layernorm<float>(y, D, a, D, M, D, nullptr, L.ln2_g, L.ln2_b, st));
  TR_TRY(gemm<float>(a, D, L.W1, H, L.b1, hbuf, H, M, H, D, EPI_RELU, st));
  TR_TRY(gemm<float>(hbuf, H, L.W2, D, L.b2, y, D, M, D, H, EPI_ACCUM, st));
  return TR_OK;
}

}  // namespace

tr_status simt_prefill(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                       cudaStream_t st) {
  const int D = m->desc.D, H = m->desc.ffn_hidden;
  if (L_u == 0) return TR_OK;
  float* ws = nullptr;
  TR_TRY(workspace((size_t)L_u * (6 * D + H) * sizeof(float), st, (void**)&ws));
  float *y = ws, *a = y + L_u * D, *qkv = a + L_u * D, *o = qkv + 3 * L_u * D, *hb = o + L_u * D;
  add_vec_rows<float><<<ceil_div((int64_t)L_u * D, 256), 256, 0, st>>>(user_tokens, y, L_u, D,
                                                                        m->domain_emb + (int64_t)domain * D);
  TR_LAUNCH_CHECK("add_vec_rows");
  const int Lp = round_up16(L_u);
  for (int l = 0; l < m->desc.n_layer; ++l) {
    void* kv_l;
    if (m->desc.dtype == TR_F32)
      kv_l = (float*)kv + (size_t)l * 2 * L_u * D;
    else
      kv_l = (__half*)kv + (size_t)l * 2 * Lp * D;
    // attention among the users reads their fp32 K/V straight from the qkv buffer
    KvF32 self_kv{qkv + D, qkv + 2 * D, 3 * D};
    TR_TRY(layer(m, l, y, a, qkv, o, hb, L_u, self_kv, L_u, 0, kv_l, st));
  }
  return TR_OK;
}

tr_status simt_compress(const tr_model* m, const void* x, int64_t n, void* tokens, cudaStream_t st) {
  const int* c = m->desc.comp_dims;
  const int64_t chunk = 16384;
  float* ws = nullptr;
  const int64_t rows = std::min<int64_t>(n, chunk);
  TR_TRY(workspace((size_t)rows * (c[1] + c[2] + c[3]) * sizeof(float), st, (void**)&ws));
  float *h1 = ws, *h2 = h1 + rows * c[1], *t = h2 + rows * c[2];
  for (int64_t r0 = 0; r0 < n; r0 += chunk) {
    const int M = (int)std::min<int64_t>(chunk, n - r0);
    if (m->desc.dtype == TR_F32)
      TR_TRY(gemm<float>((const float*)x + r0 * c[0], c[0], m->comp_W[0], c[1], m->comp_b[0], h1, c[1], M, c[1], c[0],
                         EPI_NONE, st));
    else
      TR_TRY(gemm<__nv_bfloat16>((const __nv_bfloat16*)x + r0 * c[0], c[0], m->comp_W[0], c[1], m->comp_b[0], h1,
                                 c[1], M, c[1], c[0], EPI_NONE, st));
    TR_TRY(layernorm<float>(h1, c[1], h1, c[1], M, c[1], m->comp_prelu[0], m->comp_ln_g[0], m->comp_ln_b[0], st));
    TR_TRY(gemm<float>(h1, c[1], m->comp_W[1], c[2], m->comp_b[1], h2, c[2], M, c[2], c[1], EPI_NONE, st));
    TR_TRY(layernorm<float>(h2, c[2], h2, c[2], M, c[2], m->comp_prelu[1], m->comp_ln_g[1], m->comp_ln_b[1], st));
    TR_TRY(gemm<float>(h2, c[2], m->comp_W[2], c[3], m->comp_b[2], t, c[3], M, c[3], c[2], EPI_NONE, st));
    const int64_t cnt = (int64_t)M * c[3];
    convert_rows<float><<<ceil_div(cnt, 256), 256, 0, st>>>(t, (float*)tokens + r0 * c[3], cnt);
    TR_LAUNCH_CHECK("convert_rows");
  }
  return TR_OK;
}

// Mean of each group of lt consecutive per-token scores (one candidate's tokens).
__global__ void group_mean(const float* __restrict__ x, int64_t n, int lt, float* __restrict__ out) {
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= n) return;
  float s = 0.f;
  for (int t = 0; t < lt; ++t) s += x[c * lt + t];
  out[c] = s / lt;
}

// Candidates c0 .. c1-1, each of lt tokens (rows c*lt .. c*lt+lt-1 of `tokens`): every
// token runs through the layers attending to the request's users and to its own
// candidate's lt tokens; the candidate's score is the mean of its tokens' head outputs
// (for lt = 1 the plain single-token score).
tr_status simt_score_lt(const tr_model* m, const void* tokens, bool tokens_f32, int64_t c0, int64_t c1, int lt,
                        const void* kv, int L_u, int domain, float* scores, cudaStream_t st) {
  const int D = m->desc.D, H = m->desc.ffn_hidden;
  const int64_t chunk = std::max<int64_t>(1, 16384 / lt);     // candidates per pass
  const int64_t n = c1 - c0;
  if (n <= 0) return TR_OK;
  const int64_t rows = std::min<int64_t>(n, chunk) * lt;
  float* ws = nullptr;
  TR_TRY(workspace((size_t)rows * (6 * D + H + 1) * sizeof(float), st, (void**)&ws));
  float *y = ws, *a = y + rows * D, *qkv = a + rows * D, *o = qkv + 3 * rows * D, *hb = o + rows * D;
  float* tok_scores = hb + rows * H;
  const int Lp = round_up16(L_u);
  for (int64_t q0 = c0; q0 < c1; q0 += chunk) {
    const int64_t nc = std::min<int64_t>(chunk, c1 - q0);
    const int M = (int)(nc * lt);
    const int64_t r0 = q0 * lt, cnt = (int64_t)M * D;
    if (tokens_f32)
      add_vec_rows<float><<<ceil_div(cnt, 256), 256, 0, st>>>((const float*)tokens + r0 * D, y, M, D,
                                                              m->domain_emb + (int64_t)domain * D);
    else
      add_vec_rows<__nv_bfloat16><<<ceil_div(cnt, 256), 256, 0, st>>>((const __nv_bfloat16*)tokens + r0 * D, y, M,
                                                                      D, m->domain_emb + (int64_t)domain * D);
    TR_LAUNCH_CHECK("add_vec_rows");
    for (int l = 0; l < m->desc.n_layer; ++l) {
      if (m->desc.dtype == TR_F32) {
        const float* base = (const float*)kv + (size_t)l * 2 * L_u * D;
        TR_TRY(layer(m, l, y, a, qkv, o, hb, M, KvF32{base, base + (size_t)L_u * D, D}, L_u, lt, nullptr, st));
      } else {
        const __half* base = (const __half*)kv + (size_t)l * 2 * Lp * D;
        TR_TRY(layer(m, l, y, a, qkv, o, hb, M, KvF16Image{base, base + (size_t)Lp * D, Lp, D}, L_u, lt, nullptr,
                     st));
      }
    }
    float* dst = lt == 1 ? scores + q0 : tok_scores;
    head_rows<<<ceil_div(M, 8), 256, 0, st>>>(y, M, D, m->lnf_g, m->lnf_b, m->w_head, m->b_head, dst);
    TR_LAUNCH_CHECK("head_rows");
    if (lt > 1) {
      group_mean<<<ceil_div(nc, 256), 256, 0, st>>>(tok_scores, nc, lt, scores + q0);
      TR_LAUNCH_CHECK("group_mean");
    }
  }
  return TR_OK;
}

tr_status simt_score(const tr_model* m, const void* tokens, int64_t c0, int64_t c1, const void* kv, int L_u,
                     int domain, float* scores, cudaStream_t st) {
  return simt_score_lt(m, tokens, true, c0, c1, 1, kv, L_u, domain, scores, st);
}

// ---------------------------------------------------------------- user side without allocation
// Scratch of tr_prefill_user_noalloc: a file-scope device array (every device that loads the
// library holds it until exit).  Host code only ever sees its host-side stand-in, so each
// device's address is looked up once, with that device current, and passed to the kernels.
static __device__ __align__(256) float g_noalloc_scratch[TR_NOALLOC_SCRATCH_BYTES / sizeof(float)];

tr_status simt_prefill_noalloc(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                               cudaStream_t st) {
  static std::mutex mu;
  static float* scratch_of_device[64] = {};
  const int D = m->desc.D, H = m->desc.ffn_hidden;
  const size_t need = (size_t)L_u * (6 * D + H) * sizeof(float);
  if (need > TR_NOALLOC_SCRATCH_BYTES)
    return fail(TR_ERR_INVALID_ARG,
                "tr_prefill_user_noalloc: L_u=%d needs %zu bytes of scratch, the fixed array holds %u", L_u, need,
                (unsigned)TR_NOALLOC_SCRATCH_BYTES);
  if (L_u == 0) return TR_OK;
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(TR_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  float* ws = nullptr;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!scratch_of_device[dev]) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess)
        return fail(TR_ERR_CUDA, "cudaGetSymbolAddress of the no-allocation scratch failed: %s", cudaGetErrorString(e));
      scratch_of_device[dev] = static_cast<float*>(p);
    }
    ws = scratch_of_device[dev];
  }
  float *y = ws, *a = y + L_u * D, *qkv = a + L_u * D, *o = qkv + 3 * L_u * D, *hb = o + L_u * D;
  add_vec_rows<float><<<ceil_div((int64_t)L_u * D, 256), 256, 0, st>>>(user_tokens, y, L_u, D,
                                                                        m->domain_emb + (int64_t)domain * D);
  TR_LAUNCH_CHECK("add_vec_rows");
  const int Lp = round_up16(L_u);
  for (int l = 0; l < m->desc.n_layer; ++l) {
    void* kv_l;
    if (m->desc.dtype == TR_F32)
      kv_l = (float*)kv + (size_t)l * 2 * L_u * D;
    else
      kv_l = (__half*)kv + (size_t)l * 2 * Lp * D;
    KvF32 self_kv{qkv + D, qkv + 2 * D, 3 * D};
    TR_TRY(layer(m, l, y, a, qkv, o, hb, L_u, self_kv, L_u, 0, kv_l, st));
  }
  return TR_OK;
}

}  // namespace tr
