// Per-request top-k of candidate scores: the selection step that follows scoring in GPU
// retrieval (TransRetrieval deployment section: the scored candidates of a request are
// reduced to the best few before they leave the GPU).
//
// One CTA per request.  Scores are mapped to order-preserving 32-bit keys (NaN -> the
// lowest key) and the k-th largest key is found by an MSB-first radix select, 8 bits per
// pass over the request's scores (histograms per warp in shared memory).  A final pass in
// index order keeps every score above that key and, of the scores equal to it, the ones
// with the lowest indices (a block-wide ranking), so the selected set is unique.  The k
// winners are then sorted in shared memory (bitonic, by key descending then index
// ascending) and written out.  Requests with fewer than k candidates are padded with
// index -1 and score -inf.
#include <algorithm>

#include "model.cuh"

namespace tr {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (f != f) return 0u;                                   // NaN: below everything
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkParams {
  const float* scores;
  int64_t* out_idx;
  float* out_score;
  int k, k_pow2;
  long long off[TR_MAX_REQUESTS + 1];
};

__global__ void __launch_bounds__(kThreads) topk_kernel(const __grid_constant__ TopkParams p) {
  __shared__ uint32_t hist[kWarps][256];
  __shared__ uint32_t tot[256];
  __shared__ uint32_t s_prefix, s_krem, s_sel_gt, s_warp_eq[kWarps], s_eq_base;
  extern __shared__ unsigned long long sel[];              // [k_pow2] composite sort keys
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long b0 = p.off[r], n = p.off[r + 1] - p.off[r];
  const float* sc = p.scores + b0;
  const int k = p.k;
  const int take = (int)(n < k ? n : k);

  // ---- radix select: the key of the take-th largest score and how many equal to it to keep
  uint32_t prefix = 0, mask = 0, krem = (uint32_t)take;
  if (take > 0 && take < n) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < kWarps * 256; i += kThreads) (&hist[0][0])[i] = 0u;
      __syncthreads();
      for (long long i = tid; i < n; i += kThreads) {
        const uint32_t key = order_key(__ldg(sc + i));
        if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 0xFFu], 1u);
      }
      __syncthreads();
      if (tid < 256) {
        uint32_t s = 0;
        for (int w = 0; w < kWarps; ++w) s += hist[w][tid];
        tot[tid] = s;
      }
      __syncthreads();
      if (tid == 0) {   // from the top digit down: the digit holding the krem-th largest
        uint32_t above = 0;
        int d = 255;
        for (; d > 0; --d) {
          if (above + tot[d] >= krem) break;
          above += tot[d];
        }
        s_prefix = prefix | ((uint32_t)d << shift);
        s_krem = krem - above;
      }
      __syncthreads();
      prefix = s_prefix;
      krem = s_krem;
      mask |= 0xFFu << shift;
    }
  }
  // threshold key: keep key > thr, and the krem lowest-index keys == thr
  const bool all = take == n;                    // every candidate is kept
  const uint32_t thr = prefix;
  if (tid == 0) {
    s_sel_gt = 0;
    s_eq_base = 0;
  }
  __syncthreads();
  // ---- collect in index order (chunks of kThreads); ties ranked by a block scan
  const int n_gt = all ? 0 : take - (int)krem;   // slots [0, n_gt) for keys above thr
  for (long long c0 = 0; c0 < n; c0 += kThreads) {
    const long long i = c0 + tid;
    uint32_t key = 0;
    bool gt = false, eq = false;
    if (i < n) {
      key = order_key(__ldg(sc + i));
      gt = all || key > thr;
      eq = !all && key == thr;
    }
    if (gt) {
      const uint32_t slot = atomicAdd(&s_sel_gt, 1u);
      sel[slot] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) s_warp_eq[warp] = __popc(bal);
    __syncthreads();
    uint32_t before = s_eq_base;
    for (int w = 0; w < warp; ++w) before += s_warp_eq[w];
    before += __popc(bal & ((1u << lane) - 1u));
    if (eq && before < krem) sel[n_gt + before] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
    __syncthreads();
    if (tid == 0) {
      uint32_t s = 0;
      for (int w = 0; w < kWarps; ++w) s += s_warp_eq[w];
      s_eq_base += s;
    }
    __syncthreads();
  }
  // pad to the sort size with the smallest composite key
  for (int i = take + tid; i < p.k_pow2; i += kThreads) sel[i] = 0ull;
  __syncthreads();
  // ---- bitonic sort, descending
  for (int size = 2; size <= p.k_pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < p.k_pow2; i += kThreads) {
        const int j = i ^ stride;
        if (j > i) {
          const unsigned long long a = sel[i], bb = sel[j];
          const bool desc = (i & size) == 0;
          if (desc ? (a < bb) : (a > bb)) {
            sel[i] = bb;
            sel[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // ---- write out
  for (int j = tid; j < k; j += kThreads) {
    int64_t idx = -1;
    float v = -INFINITY;
    if (j < take) {
      const unsigned long long c = sel[j];
      idx = (int64_t)(0xFFFFFFFFu - (uint32_t)(c & 0xFFFFFFFFull));
      v = __ldg(sc + idx);
    }
    p.out_idx[(size_t)r * k + j] = idx;
    if (p.out_score) p.out_score[(size_t)r * k + j] = v;
  }
}

}  // namespace

tr_status launch_topk(const float* scores, const int64_t* req_offsets, int R, int k, int64_t* out_idx,
                      float* out_score, cudaStream_t st) {
  TopkParams p{};
  p.scores = scores;
  p.out_idx = out_idx;
  p.out_score = out_score;
  p.k = k;
  int kp = 1;
  while (kp < k) kp <<= 1;
  p.k_pow2 = kp;
  for (int r = 0; r <= R; ++r) p.off[r] = req_offsets[r];
  const size_t smem = (size_t)kp * sizeof(unsigned long long);
  static bool attr_set[64] = {};
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    TR_CUDA_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)(TR_MAX_TOPK * sizeof(unsigned long long))));
    attr_set[dev] = true;
  }
  topk_kernel<<<R, kThreads, smem, st>>>(p);
  TR_LAUNCH_CHECK("topk_kernel");
  return TR_OK;
}

}  // namespace tr
