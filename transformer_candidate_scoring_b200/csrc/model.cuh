// Device-resident model: fp32 copies in the layouts of the C ABI plus, for bf16 models,
// the repacked operand images the tensor-core kernels read.
#pragma once

#include <vector>

#include "common.cuh"

struct tr_layer_dev {
  const float *ln1_g, *ln1_b, *Wqkv, *bqkv, *Wo, *bo, *ln2_g, *ln2_b, *W1, *b1, *W2, *b2;
};

struct tr_model {
  tr_model_desc desc;
  int device;
  float* f32_blob = nullptr;            // all fp32 parameters, one allocation
  const float* domain_emb = nullptr;    // [n_domains][D]
  std::vector<tr_layer_dev> layers;     // Wqkv is [D][3D] (q | k | v columns), bqkv [3D]
  const float *lnf_g = nullptr, *lnf_b = nullptr, *w_head = nullptr;
  float b_head = 0.f;
  const float* comp_W[3] = {};
  const float* comp_b[3] = {};
  const float* comp_prelu[2] = {};
  const float* comp_ln_g[2] = {};
  const float* comp_ln_b[2] = {};

  // tensor-core operand images (bf16 models only; null until built)
  void* tc_blob = nullptr;
  size_t tc_bytes = 0;
  const void* tc_stack = nullptr;       // per-layer weight images of the candidate stack
  size_t tc_stack_layer_bytes = 0;
  const float* tc_vec = nullptr;        // folded bias / gain vectors of the candidate stack
  size_t tc_vec_layer_floats = 0;
  const void* tc_comp = nullptr;        // compressor operand images
  const float* tc_comp_vec = nullptr;
};

namespace tr {
// SIMT path (any dtype; fp32 arithmetic)
tr_status simt_prefill(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv,
                       cudaStream_t st);
tr_status simt_compress(const tr_model* m, const void* x, int64_t n, void* tokens, cudaStream_t st);
tr_status simt_score(const tr_model* m, const void* tokens, int64_t c0, int64_t c1, const void* kv,
                     int L_u, int domain, float* scores, cudaStream_t st);   // fp32 tokens
tr_status simt_score_lt(const tr_model* m, const void* tokens, bool tokens_f32, int64_t c0, int64_t c1, int lt,
                        const void* kv, int L_u, int domain, float* scores, cudaStream_t st);
tr_status launch_topk(const float* scores, const int64_t* req_offsets, int R, int k, int64_t* out_idx,
                      float* out_score, cudaStream_t st);
tr_status launch_aggregate(const tr_table* tables, int n_tables, const int32_t* bag_table,
                           const int64_t* offsets, const int32_t* keys, const float* weights,
                           int64_t n_bags, int D, tr_dtype out_dtype, int mode, void* out, cudaStream_t st);
}  // namespace tr
