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
constexpr int kUnroll = 8;   // score loads in flight per thread

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
  __shared__ uint32_t s_prefix, s_krem, s_sel_gt, s_warp_eq[kWarps], s_eq_base, s_eq_total;
  extern __shared__ unsigned long long sel[];              // [k_pow2] composite sort keys
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long b0 = p.off[r], n = p.off[r + 1] - p.off[r];
  const float* sc = p.scores + b0;
  const int k = p.k;
  const int take = (int)(n < k ? n : k);
  const int n32 = (int)n;

  // ---- radix select: the key of the take-th largest score and how many equal to it to keep
  uint32_t prefix = 0, mask = 0, krem = (uint32_t)take;
  if (take > 0 && take < n) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < kWarps * 256; i += kThreads) (&hist[0][0])[i] = 0u;
      __syncthreads();
      // eight loads in flight per thread; 32-bit indices (a request has < 2^31 candidates)
      for (int i0 = 0; i0 < n32; i0 += kThreads * kUnroll) {
        uint32_t key[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int i = i0 + u * kThreads + tid;
          key[u] = i < n32 ? order_key(__ldg(sc + i)) : 0u;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int i = i0 + u * kThreads + tid;
          if (i < n32 && (key[u] & mask) == prefix) atomicAdd(&hist[warp][(key[u] >> shift) & 0xFFu], 1u);
        }
      }
      __syncthreads();
      // bin totals from the top digit down, as an inclusive scan over 256 threads: thread t
      // holds digit 255 - t, and the digit whose running count first reaches krem wins
      __shared__ uint32_t s_wsum[8];
      uint32_t cnt = 0, incl = 0;
      if (tid < 256) {
        const int d = 255 - tid;
        for (int w = 0; w < kWarps; ++w) cnt += hist[w][d];
        incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        if (lane == 31) s_wsum[warp] = incl;
      }
      __syncthreads();
      if (tid < 256) {
        for (int w = 0; w < warp; ++w) incl += s_wsum[w];
        const uint32_t excl = incl - cnt;
        if (excl < krem && krem <= incl) {
          s_prefix = prefix | ((uint32_t)(255 - tid) << shift);
          s_krem = krem - excl;
          s_eq_total = cnt;   // after the last pass: how many scores equal the threshold
        }
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
  // ---- collect.  When every score equal to the threshold is kept (always, unless ties
  // straddle the k-th place) one unordered pass suffices; otherwise the equal scores are
  // ranked by index with a block scan, chunk by chunk in index order.
  const int n_gt = all ? 0 : take - (int)krem;   // slots [0, n_gt) for keys above thr
  const bool keep_all_eq = all || s_eq_total == krem;
  for (int g0 = 0; keep_all_eq && g0 < n32; g0 += kThreads * kUnroll) {
    uint32_t keys[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = g0 + u * kThreads + tid;
      keys[u] = i < n32 ? order_key(__ldg(sc + i)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = g0 + u * kThreads + tid;
      const bool in = i < n32 && (all || keys[u] >= thr);
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      uint32_t base = 0;
      if (lane == 0 && bal) base = atomicAdd(&s_sel_gt, (uint32_t)__popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (in) sel[base + __popc(bal & ((1u << lane) - 1u))] = ((unsigned long long)keys[u] << 32) | (0xFFFFFFFFu - (uint32_t)i);
    }
  }
  for (long long g0 = 0; !keep_all_eq && g0 < n; g0 += (long long)kThreads * kUnroll) {
    uint32_t keys[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {   // the loads of eight chunks first
      const long long i = g0 + (long long)u * kThreads + tid;
      keys[u] = i < n ? order_key(__ldg(sc + i)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {   // then the chunks in index order
      const long long c0 = g0 + (long long)u * kThreads;
      if (c0 >= n) break;
      const long long i = c0 + tid;
      const uint32_t key = keys[u];
      const bool gt = i < n && (all || key > thr);
      const bool eq = i < n && !all && key == thr;
      const unsigned bal_gt = __ballot_sync(0xffffffffu, gt);   // one slot reservation per warp
      uint32_t base = 0;
      if (lane == 0 && bal_gt) base = atomicAdd(&s_sel_gt, (uint32_t)__popc(bal_gt));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (gt) sel[base + __popc(bal_gt & ((1u << lane) - 1u))] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      if (lane == 0) s_warp_eq[warp] = __popc(bal);
      __syncthreads();
      uint32_t before = s_eq_base;
      for (int w = 0; w < warp; ++w) before += s_warp_eq[w];
      before += __popc(bal & ((1u << lane) - 1u));
      if (eq && before < krem) sel[n_gt + before] = ((unsigned long long)key << 32) | (0xFFFFFFFFu - (uint32_t)i);
      __syncthreads();
      if (tid == 0) {
        uint32_t t = 0;
        for (int w = 0; w < kWarps; ++w) t += s_warp_eq[w];
        s_eq_base += t;
      }
      __syncthreads();
    }
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
  TR_TRY(ensure_smem_attr((const void*)topk_kernel, (int)(TR_MAX_TOPK * sizeof(unsigned long long))));
  topk_kernel<<<R, kThreads, smem, st>>>(p);
  TR_LAUNCH_CHECK("topk_kernel");
  return TR_OK;
}

}  // namespace tr
