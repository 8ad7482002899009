// C ABI of libtr: argument validation, model construction, dispatch to the kernels.
#include <stdarg.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <mutex>
#include <thread>
#include <vector>

#include "model.cuh"

namespace tr {

static thread_local std::string g_err;

void set_error(const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
}

tr_status fail(tr_status code, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static std::mutex g_dev_mu;
static DeviceState g_dev[64];

tr_status device_state(DeviceState** out) {
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(TR_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceState& s = g_dev[dev];
  if (!s.status) {
    TR_CUDA_TRY(cudaMalloc(&s.status, sizeof(int)));
    TR_CUDA_TRY(cudaMemset(s.status, 0, sizeof(int)));
  }
  *out = &s;
  return TR_OK;
}

namespace {
struct StreamScratch {
  int dev;
  cudaStream_t stream;
  void* ptr;
  size_t bytes;
};
std::vector<StreamScratch> g_scratch;   // guarded by g_dev_mu
std::vector<std::pair<int, const void*>> g_attr_done;
}  // namespace

tr_status workspace(size_t bytes, cudaStream_t st, void** out) {
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  StreamScratch* s = nullptr;
  for (auto& e : g_scratch)
    if (e.dev == dev && e.stream == st) s = &e;
  if (!s) {
    g_scratch.push_back({dev, st, nullptr, 0});
    s = &g_scratch.back();
  }
  if (s->bytes < bytes) {
    if (s->ptr) {
      // earlier work on this stream may still read the old buffer
      TR_CUDA_TRY(cudaStreamSynchronize(st));
      TR_CUDA_TRY(cudaFree(s->ptr));
      s->ptr = nullptr;
      s->bytes = 0;
    }
    const size_t want = bytes + bytes / 4;
    if (cudaMalloc(&s->ptr, want) != cudaSuccess) {
      cudaGetLastError();
      s->ptr = nullptr;
      return fail(TR_ERR_NOMEM, "workspace allocation of %zu bytes failed", want);
    }
    s->bytes = want;
  }
  *out = s->ptr;
  return TR_OK;
}

namespace {
struct StreamInts {
  int dev;
  cudaStream_t stream;
  int* ptr;
};
std::vector<StreamInts> g_counters;   // guarded by g_dev_mu
}  // namespace

tr_status stream_counters(cudaStream_t st, int** out) {
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  for (auto& e : g_counters)
    if (e.dev == dev && e.stream == st) {
      *out = e.ptr;
      return TR_OK;
    }
  int* p = nullptr;
  if (cudaMalloc(&p, 64 * sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return fail(TR_ERR_NOMEM, "stream counters: allocation failed");
  }
  TR_CUDA_TRY(cudaMemset(p, 0, 64 * sizeof(int)));
  g_counters.push_back({dev, st, p});
  *out = p;
  return TR_OK;
}

tr_status ensure_smem_attr(const void* kernel, int bytes) {
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  for (auto& e : g_attr_done)
    if (e.first == dev && e.second == kernel) return TR_OK;
  TR_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  g_attr_done.push_back({dev, kernel});
  return TR_OK;
}

// tensor-core stack / compressor (defined in their own translation units)
tr_status tc_build(tr_model* m, const tr_model_weights* w);
bool tc_stack_supported(const tr_model* m);
tr_status tc_score(const tr_model* m, const void* tokens, int64_t n, const int64_t* req_offsets,
                   const void* const* kv, const int32_t* L_u, const int32_t* domain, int R, float* scores,
                   cudaStream_t st);
bool tc_comp_supported(const tr_model* m);
tr_status tc_compress(const tr_model* m, const void* x, int64_t n, void* tokens, cudaStream_t st);
bool tc_comp_bags_supported(const tr_model* m);
bool tc_score_lt_supported(const tr_model* m, int L_t, const int32_t* L_u, int R);
tr_status tc_score_lt(const tr_model* m, const void* tokens, int L_t, const int64_t* req_offsets,
                      const void* const* kv, const int32_t* L_u, const int32_t* domain, int R, float* scores,
                      cudaStream_t st);
tr_status tc_compress_bags(const tr_model* m, const tr_table* tables, int n_tables, const int32_t* bag_table,
                           const int64_t* offsets, const int32_t* keys, const float* weights, int64_t n,
                           void* tokens, cudaStream_t st);
bool tc_prefill_supported(const tr_model* m, int L_u);
tr_status simt_prefill_noalloc(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                               cudaStream_t st);
tr_status tc_prefill(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv, cudaStream_t st);
tr_status tc_prefill_batch(const tr_model* m, const float* const* user_tokens, const int32_t* L_u,
                           const int32_t* domain, void* const* kv, int R, cudaStream_t st);

}  // namespace tr

using namespace tr;

extern "C" {

const char* tr_last_error(void) { return g_err.c_str(); }
const char* tr_version(void) { return "libtr 0.1 (sm_100a)"; }
unsigned long long tr_kernel_launches(void) { return g_launches.load(); }

static tr_status validate_desc(const tr_model_desc* d) {
  if (!d) return fail(TR_ERR_INVALID_ARG, "desc is null");
  if (d->D <= 0 || d->D % 16 || d->D > 128) return fail(TR_ERR_UNSUPPORTED, "D=%d: need a multiple of 16 <= 128", d->D);
  if (d->n_layer < 1 || d->n_layer > 16) return fail(TR_ERR_UNSUPPORTED, "n_layer=%d: need 1..16", d->n_layer);
  if (d->n_head <= 0 || d->D % d->n_head || d->D / d->n_head != kDHead)
    return fail(TR_ERR_UNSUPPORTED, "D/n_head must be %d (D=%d, n_head=%d)", kDHead, d->D, d->n_head);
  if (d->ffn_hidden <= 0 || d->ffn_hidden % 16 || d->ffn_hidden > 512)
    return fail(TR_ERR_UNSUPPORTED, "ffn_hidden=%d: need a multiple of 16 <= 512", d->ffn_hidden);
  if (d->n_target_fields <= 0) return fail(TR_ERR_INVALID_ARG, "n_target_fields=%d", d->n_target_fields);
  if (d->comp_dims[0] != d->n_target_fields * d->D)
    return fail(TR_ERR_INVALID_ARG, "comp_dims[0]=%d must equal F*D=%d", d->comp_dims[0], d->n_target_fields * d->D);
  if (d->comp_dims[3] != d->D) return fail(TR_ERR_INVALID_ARG, "comp_dims[3]=%d must equal D", d->comp_dims[3]);
  for (int i = 0; i < 4; ++i)
    if (d->comp_dims[i] <= 0 || d->comp_dims[i] % 16 || d->comp_dims[i] > 4096)
      return fail(TR_ERR_UNSUPPORTED, "comp_dims[%d]=%d: need a multiple of 16 <= 4096", i, d->comp_dims[i]);
  if (d->n_domains <= 0) return fail(TR_ERR_INVALID_ARG, "n_domains=%d", d->n_domains);
  if (d->dtype != TR_F32 && d->dtype != TR_BF16) return fail(TR_ERR_INVALID_ARG, "dtype=%d", (int)d->dtype);
  return TR_OK;
}

tr_status tr_model_create(const tr_model_desc* desc, const tr_model_weights* w, tr_model** out) {
  if (out) *out = nullptr;
  TR_TRY(validate_desc(desc));
  if (!w || !out || !w->layers) return fail(TR_ERR_INVALID_ARG, "null weights/out/layers");
  const int D = desc->D, H = desc->ffn_hidden, N = desc->n_layer;
  const int* c = desc->comp_dims;
  // host staging of every fp32 parameter, in blob order
  std::vector<float> blob;
  std::vector<size_t> offs;
  auto push = [&](const float* p, size_t n) -> bool {
    if (!p) return false;
    offs.push_back(blob.size());
    blob.insert(blob.end(), p, p + n);
    while (blob.size() % 64) blob.push_back(0.f);  // 256-byte alignment of every tensor
    return true;
  };
  bool ok = push(w->domain_emb, (size_t)desc->n_domains * D);
  std::vector<float> wqkv((size_t)D * 3 * D), bqkv(3 * D);
  for (int l = 0; l < N && ok; ++l) {
    const tr_layer_weights& L = w->layers[l];
    if (!L.Wq || !L.Wk || !L.Wv || !L.bq || !L.bk || !L.bv) { ok = false; break; }
    for (int i = 0; i < D; ++i)
      for (int j = 0; j < D; ++j) {
        wqkv[(size_t)i * 3 * D + j] = L.Wq[(size_t)i * D + j];
        wqkv[(size_t)i * 3 * D + D + j] = L.Wk[(size_t)i * D + j];
        wqkv[(size_t)i * 3 * D + 2 * D + j] = L.Wv[(size_t)i * D + j];
      }
    for (int j = 0; j < D; ++j) { bqkv[j] = L.bq[j]; bqkv[D + j] = L.bk[j]; bqkv[2 * D + j] = L.bv[j]; }
    ok = push(L.ln1_g, D) && push(L.ln1_b, D) && push(wqkv.data(), wqkv.size()) && push(bqkv.data(), bqkv.size()) &&
         push(L.Wo, (size_t)D * D) && push(L.bo, D) && push(L.ln2_g, D) && push(L.ln2_b, D) &&
         push(L.W1, (size_t)D * H) && push(L.b1, H) && push(L.W2, (size_t)H * D) && push(L.b2, D);
  }
  ok = ok && push(w->lnf_g, D) && push(w->lnf_b, D) && push(w->w_head, D);
  for (int i = 0; i < 3 && ok; ++i) ok = push(w->comp_W[i], (size_t)c[i] * c[i + 1]) && push(w->comp_b[i], c[i + 1]);
  for (int i = 0; i < 2 && ok; ++i)
    ok = push(w->comp_prelu[i], c[i + 1]) && push(w->comp_ln_g[i], c[i + 1]) && push(w->comp_ln_b[i], c[i + 1]);
  if (!ok) return fail(TR_ERR_INVALID_ARG, "a weight pointer is null");

  tr_model* m = new tr_model();
  m->desc = *desc;
  if (cudaGetDevice(&m->device) != cudaSuccess ||
      cudaMalloc(&m->f32_blob, blob.size() * sizeof(float)) != cudaSuccess) {
    cudaGetLastError();
    delete m;
    return fail(TR_ERR_NOMEM, "model allocation failed");
  }
  if (cudaMemcpy(m->f32_blob, blob.data(), blob.size() * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(m->f32_blob);
    delete m;
    return fail(TR_ERR_CUDA, "model upload failed");
  }
  size_t k = 0;
  auto nxt = [&]() { return (const float*)m->f32_blob + offs[k++]; };
  m->domain_emb = nxt();
  m->layers.resize(N);
  for (int l = 0; l < N; ++l) {
    tr_layer_dev& L = m->layers[l];
    L.ln1_g = nxt(); L.ln1_b = nxt(); L.Wqkv = nxt(); L.bqkv = nxt(); L.Wo = nxt(); L.bo = nxt();
    L.ln2_g = nxt(); L.ln2_b = nxt(); L.W1 = nxt(); L.b1 = nxt(); L.W2 = nxt(); L.b2 = nxt();
  }
  m->lnf_g = nxt(); m->lnf_b = nxt(); m->w_head = nxt();
  m->b_head = w->b_head;
  for (int i = 0; i < 3; ++i) { m->comp_W[i] = nxt(); m->comp_b[i] = nxt(); }
  for (int i = 0; i < 2; ++i) { m->comp_prelu[i] = nxt(); m->comp_ln_g[i] = nxt(); m->comp_ln_b[i] = nxt(); }
  const char* force = getenv("TR_FORCE_SIMT");
  if (desc->dtype == TR_BF16 && !(force && force[0] == '1')) {
    tr_status s = tc_build(m, w);
    if (s != TR_OK) {
      tr_model_destroy(m);
      return s;
    }
  }
  *out = m;
  return TR_OK;
}

void tr_model_destroy(tr_model* m) {
  if (!m) return;
  int prev = 0;
  cudaGetDevice(&prev);
  cudaSetDevice(m->device);
  if (m->f32_blob) cudaFree(m->f32_blob);
  if (m->tc_blob) cudaFree(m->tc_blob);
  if (m->tc_comp) cudaFree(const_cast<void*>(m->tc_comp));
  cudaSetDevice(prev);
  delete m;
}

static tr_status check_model_device(const tr_model* m) {
  if (!m) return fail(TR_ERR_INVALID_ARG, "model is null");
  int dev = -1;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  if (dev != m->device) return fail(TR_ERR_INVALID_ARG, "model lives on device %d, current device is %d", m->device, dev);
  return TR_OK;
}

tr_status tr_aggregate(const tr_table* tables, int n_tables, const int32_t* bag_table, const int64_t* offsets,
                       const int32_t* keys, const float* weights, int64_t n_bags, int D, tr_dtype out_dtype,
                       void* out, tr_stream stream) {
  return tr_aggregate_ex(tables, n_tables, bag_table, offsets, keys, weights, n_bags, D, out_dtype, TR_AGG_MEAN,
                         out, stream);
}

tr_status tr_aggregate_ex(const tr_table* tables, int n_tables, const int32_t* bag_table, const int64_t* offsets,
                          const int32_t* keys, const float* weights, int64_t n_bags, int D, tr_dtype out_dtype,
                          int mode, void* out, tr_stream stream) {
  const int agg = mode & ~TR_AGG_POST_LN;
  if (agg != TR_AGG_MEAN && agg != TR_AGG_SUM && agg != TR_AGG_MAX)
    return fail(TR_ERR_INVALID_ARG, "aggregation mode %d", mode);
  if (n_bags < 0) return fail(TR_ERR_INVALID_ARG, "n_bags=%lld", (long long)n_bags);
  if (n_bags == 0) return TR_OK;
  if (!tables || n_tables <= 0 || n_tables > TR_MAX_TABLES)
    return fail(TR_ERR_INVALID_ARG, "n_tables=%d (need 1..%d) or tables null", n_tables, TR_MAX_TABLES);
  if (!bag_table || !offsets || !keys || !weights || !out) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  if (D <= 0 || D % 8 || D > 512) return fail(TR_ERR_INVALID_ARG, "D=%d: need a multiple of 8 <= 512", D);
  if (out_dtype != TR_F32 && out_dtype != TR_BF16) return fail(TR_ERR_INVALID_ARG, "out_dtype=%d", (int)out_dtype);
  for (int i = 0; i < n_tables; ++i) {
    if (!tables[i].data || tables[i].n_rows <= 0) return fail(TR_ERR_INVALID_ARG, "table %d is empty or null", i);
    if (tables[i].dtype != tables[0].dtype) return fail(TR_ERR_INVALID_ARG, "tables must share one dtype");
    if ((uintptr_t)tables[i].data % 16) return fail(TR_ERR_INVALID_ARG, "table %d is not 16-byte aligned", i);
  }
  if ((uintptr_t)out % 16) return fail(TR_ERR_INVALID_ARG, "out is not 16-byte aligned");
  return launch_aggregate(tables, n_tables, bag_table, offsets, keys, weights, n_bags, D, out_dtype, mode, out,
                          (cudaStream_t)stream);
}

size_t tr_kv_cache_bytes(const tr_model* m, int L_u) {
  if (!m || L_u < 0 || L_u > TR_MAX_LU) return 0;
  const size_t D = m->desc.D, N = m->desc.n_layer;
  if (m->desc.dtype == TR_F32) return N * 2 * (size_t)L_u * D * sizeof(float);
  return N * 2 * (size_t)round_up16(L_u) * D * 2;
}

tr_status tr_prefill_user(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                          tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (L_u < 0 || L_u > TR_MAX_LU) return fail(TR_ERR_INVALID_ARG, "L_u=%d (need 0..%d)", L_u, TR_MAX_LU);
  if (domain < 0 || domain >= m->desc.n_domains) return fail(TR_ERR_INVALID_ARG, "domain=%d", domain);
  if (L_u == 0) return TR_OK;
  if (!user_tokens || !kv) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  if (tc_prefill_supported(m, L_u)) return tc_prefill(m, user_tokens, L_u, domain, kv, (cudaStream_t)stream);
  return simt_prefill(m, user_tokens, L_u, domain, kv, (cudaStream_t)stream);
}

tr_status tr_prefill_users(const tr_model* m, const float* const* user_tokens, const int32_t* L_u,
                           const int32_t* domain, void* const* kv, int R, tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (R < 1 || R > TR_MAX_REQUESTS) return fail(TR_ERR_INVALID_ARG, "R=%d (need 1..%d)", R, TR_MAX_REQUESTS);
  if (!user_tokens || !L_u || !domain || !kv) return fail(TR_ERR_INVALID_ARG, "null host array");
  bool batch = true;
  for (int r = 0; r < R; ++r) {
    if (L_u[r] < 0 || L_u[r] > TR_MAX_LU) return fail(TR_ERR_INVALID_ARG, "L_u[%d]=%d (need 0..%d)", r, L_u[r], TR_MAX_LU);
    if (domain[r] < 0 || domain[r] >= m->desc.n_domains) return fail(TR_ERR_INVALID_ARG, "domain[%d]=%d", r, domain[r]);
    if (L_u[r] > 0 && (!user_tokens[r] || !kv[r])) return fail(TR_ERR_INVALID_ARG, "request %d: null device pointer", r);
    batch = batch && (L_u[r] == 0 || tc_prefill_supported(m, L_u[r]));
  }
  const cudaStream_t st = (cudaStream_t)stream;
  if (batch) return tc_prefill_batch(m, user_tokens, L_u, domain, kv, R, st);
  for (int r = 0; r < R; ++r)
    if (L_u[r] > 0) TR_TRY(tr_prefill_user(m, user_tokens[r], L_u[r], domain[r], kv[r], stream));
  return TR_OK;
}

tr_status tr_prefill_user_noalloc(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                                  tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (L_u < 0 || L_u > TR_MAX_LU) return fail(TR_ERR_INVALID_ARG, "L_u=%d (need 0..%d)", L_u, TR_MAX_LU);
  if (domain < 0 || domain >= m->desc.n_domains) return fail(TR_ERR_INVALID_ARG, "domain=%d", domain);
  if (L_u > 0 && (!user_tokens || !kv)) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  return simt_prefill_noalloc(m, user_tokens, L_u, domain, kv, (cudaStream_t)stream);
}

tr_status tr_compress_targets(const tr_model* m, const void* x, int64_t n, void* tokens, tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (n < 0) return fail(TR_ERR_INVALID_ARG, "n=%lld", (long long)n);
  if (n == 0) return TR_OK;
  if (!x || !tokens) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  if (m->desc.dtype == TR_BF16 && tc_comp_supported(m))
    return tc_compress(m, x, n, tokens, (cudaStream_t)stream);
  return simt_compress(m, x, n, tokens, (cudaStream_t)stream);
}

tr_status tr_compress_target_bags(const tr_model* m, const tr_table* tables, int n_tables, const int32_t* bag_table,
                                  const int64_t* offsets, const int32_t* keys, const float* weights, int64_t n,
                                  void* tokens, tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (n < 0) return fail(TR_ERR_INVALID_ARG, "n=%lld", (long long)n);
  if (!tables || n_tables <= 0 || n_tables > TR_MAX_TABLES)
    return fail(TR_ERR_INVALID_ARG, "n_tables=%d (need 1..%d) or tables null", n_tables, TR_MAX_TABLES);
  for (int i = 0; i < n_tables; ++i) {
    if (!tables[i].data || tables[i].n_rows <= 0) return fail(TR_ERR_INVALID_ARG, "table %d is empty or null", i);
    if (tables[i].dtype != TR_BF16) return fail(TR_ERR_INVALID_ARG, "table %d is not bf16", i);
    if ((uintptr_t)tables[i].data % 16) return fail(TR_ERR_INVALID_ARG, "table %d is not 16-byte aligned", i);
  }
  if (!(m->desc.dtype == TR_BF16 && tc_comp_bags_supported(m)))
    return fail(TR_ERR_UNSUPPORTED,
                "tr_compress_target_bags needs a bf16 model on the tensor-core compressor with D a multiple of 64");
  if (n == 0) return TR_OK;
  if (!bag_table || !offsets || !keys || !weights || !tokens) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  if ((n + 127) / 128 > INT32_MAX) return fail(TR_ERR_INVALID_ARG, "n=%lld is too large", (long long)n);
  return tc_compress_bags(m, tables, n_tables, bag_table, offsets, keys, weights, n, tokens, (cudaStream_t)stream);
}

tr_status tr_score_candidates(const tr_model* m, const void* tokens, int64_t n, const int64_t* req_offsets,
                              const void* const* kv, const int32_t* L_u, const int32_t* domain, int R,
                              float* scores, tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (R < 1 || R > TR_MAX_REQUESTS) return fail(TR_ERR_INVALID_ARG, "R=%d (need 1..%d)", R, TR_MAX_REQUESTS);
  if (!req_offsets || !kv || !L_u || !domain) return fail(TR_ERR_INVALID_ARG, "null host array");
  if (n < 0 || req_offsets[0] != 0 || req_offsets[R] != n)
    return fail(TR_ERR_INVALID_ARG, "req_offsets must run from 0 to n=%lld", (long long)n);
  for (int r = 0; r < R; ++r) {
    if (req_offsets[r + 1] < req_offsets[r]) return fail(TR_ERR_INVALID_ARG, "req_offsets decrease at %d", r);
    if (L_u[r] < 0 || L_u[r] > TR_MAX_LU) return fail(TR_ERR_INVALID_ARG, "L_u[%d]=%d", r, L_u[r]);
    if (domain[r] < 0 || domain[r] >= m->desc.n_domains) return fail(TR_ERR_INVALID_ARG, "domain[%d]=%d", r, domain[r]);
    if (L_u[r] > 0 && req_offsets[r + 1] > req_offsets[r] && !kv[r])
      return fail(TR_ERR_INVALID_ARG, "kv[%d] is null", r);
  }
  if (n == 0) return TR_OK;
  if (!tokens || !scores) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  const cudaStream_t st = (cudaStream_t)stream;
  if (m->desc.dtype == TR_BF16 && tc_stack_supported(m))
    return tc_score(m, tokens, n, req_offsets, kv, L_u, domain, R, scores, st);
  for (int r = 0; r < R; ++r)
    TR_TRY(simt_score(m, tokens, req_offsets[r], req_offsets[r + 1], kv[r], L_u[r], domain[r], scores, st));
  return TR_OK;
}

tr_status tr_score_candidates_uncompressed(const tr_model* m, const void* tokens, int64_t n, int L_t,
                                           const int64_t* req_offsets, const void* const* kv, const int32_t* L_u,
                                           const int32_t* domain, int R, float* scores, tr_stream stream) {
  TR_TRY(check_model_device(m));
  if (L_t < 1 || L_t > TR_MAX_LT) return fail(TR_ERR_INVALID_ARG, "L_t=%d (need 1..%d)", L_t, TR_MAX_LT);
  if (R < 1 || R > TR_MAX_REQUESTS) return fail(TR_ERR_INVALID_ARG, "R=%d (need 1..%d)", R, TR_MAX_REQUESTS);
  if (!req_offsets || !kv || !L_u || !domain) return fail(TR_ERR_INVALID_ARG, "null host array");
  if (n < 0 || req_offsets[0] != 0 || req_offsets[R] != n)
    return fail(TR_ERR_INVALID_ARG, "req_offsets must run from 0 to n=%lld", (long long)n);
  for (int r = 0; r < R; ++r) {
    if (req_offsets[r + 1] < req_offsets[r]) return fail(TR_ERR_INVALID_ARG, "req_offsets decrease at %d", r);
    if (L_u[r] < 0 || L_u[r] > TR_MAX_LU) return fail(TR_ERR_INVALID_ARG, "L_u[%d]=%d", r, L_u[r]);
    if (domain[r] < 0 || domain[r] >= m->desc.n_domains) return fail(TR_ERR_INVALID_ARG, "domain[%d]=%d", r, domain[r]);
    if (L_u[r] > 0 && req_offsets[r + 1] > req_offsets[r] && !kv[r])
      return fail(TR_ERR_INVALID_ARG, "kv[%d] is null", r);
  }
  if (n == 0) return TR_OK;
  if (!tokens || !scores) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  const cudaStream_t st = (cudaStream_t)stream;
  if (tc_score_lt_supported(m, L_t, L_u, R)) return tc_score_lt(m, tokens, L_t, req_offsets, kv, L_u, domain, R, scores, st);
  for (int r = 0; r < R; ++r)
    TR_TRY(simt_score_lt(m, tokens, m->desc.dtype == TR_F32, req_offsets[r], req_offsets[r + 1], L_t, kv[r], L_u[r],
                         domain[r], scores, st));
  return TR_OK;
}

tr_status tr_topk(const float* scores, int64_t n, const int64_t* req_offsets, int R, int k, int64_t* out_idx,
                  float* out_score, tr_stream stream) {
  if (R < 1 || R > TR_MAX_REQUESTS) return fail(TR_ERR_INVALID_ARG, "R=%d (need 1..%d)", R, TR_MAX_REQUESTS);
  if (k < 1 || k > TR_MAX_TOPK) return fail(TR_ERR_INVALID_ARG, "k=%d (need 1..%d)", k, TR_MAX_TOPK);
  if (!req_offsets) return fail(TR_ERR_INVALID_ARG, "null req_offsets");
  if (n < 0 || req_offsets[0] != 0 || req_offsets[R] != n)
    return fail(TR_ERR_INVALID_ARG, "req_offsets must run from 0 to n=%lld", (long long)n);
  for (int r = 0; r < R; ++r) {
    if (req_offsets[r + 1] < req_offsets[r]) return fail(TR_ERR_INVALID_ARG, "req_offsets decrease at %d", r);
    if (req_offsets[r + 1] - req_offsets[r] >= (int64_t)1 << 31)
      return fail(TR_ERR_UNSUPPORTED, "request %d has 2^31 or more candidates", r);
  }
  if (!out_idx || (n > 0 && !scores)) return fail(TR_ERR_INVALID_ARG, "null device pointer");
  return launch_topk(scores, req_offsets, R, k, out_idx, out_score, (cudaStream_t)stream);
}

tr_status tr_sync_status(tr_stream stream, int timeout_ms) {
  const cudaStream_t st = (cudaStream_t)stream;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    cudaError_t e = cudaStreamQuery(st);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return fail(TR_ERR_CUDA, "stream error: %s", cudaGetErrorString(e));
    if (timeout_ms > 0 && std::chrono::steady_clock::now() - t0 > std::chrono::milliseconds(timeout_ms))
      return fail(TR_ERR_TIMEOUT, "stream did not drain within %d ms", timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  int h = 0;
  TR_CUDA_TRY(cudaMemcpy(&h, ds->status, sizeof(int), cudaMemcpyDeviceToHost));
  if (h) {
    TR_CUDA_TRY(cudaMemset(ds->status, 0, sizeof(int)));
    if (h & STATUS_KERNEL_TIMEOUT)
      return fail(TR_ERR_TIMEOUT, "a kernel gave up waiting on an internal barrier and unwound");
    if (h & STATUS_KEY_RANGE) return fail(TR_ERR_KEY_RANGE, "a key or table index was out of range (skipped)");
  }
  return TR_OK;
}

}  // extern "C"
