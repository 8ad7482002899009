// Weighted-average aggregation of (key, weight) bags (TransRetrieval §3.2):
//   out[b] = sum_i v_i h(k_i) / sum_i v_i
//
// HBM-bound gather.  A table row is split into 16-byte vectors and `LPR` lanes cover one
// row (16 lanes for a 256-byte row, D = 128 bf16).  Two kernels share the arithmetic:
//  - wavg_kernel, for many bags: each group of LPR lanes owns one bag at a time (a warp
//    works on 32 / LPR bags), with several rows in flight per group;
//  - wavg_split_kernel, for few bags (fewer than one resident round of blocks): one block
//    per bag, its 256 / LPR lane groups share the bag's rows and their partial sums meet
//    in shared memory, so a long bag costs one round of row loads instead of many.
// Keys and weights are fetched LPR at a time and broadcast by shuffle.  Accumulation is
// fp32 (packed fp32x2 FMAs); the mean multiplies by a correctly rounded reciprocal of the
// weight sum, so scaling all weights of a bag by 2^k leaves the result bit-identical.
#include <algorithm>

#include "model.cuh"

namespace tr {
namespace {

struct TableSet {
  const void* ptr[TR_MAX_TABLES];
  int64_t rows[TR_MAX_TABLES];
};

template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

// a0 += w * x0, a1 += w * x1 as one packed fp32x2 FMA (each lane rounded as fmaf)
__device__ __forceinline__ void fma2(float& a0, float& a1, float w, float x0, float x1) {
  asm("{\n\t.reg .b64 a, x, w;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 x, {%3, %4};\n\tmov.b64 w, {%2, %2};\n\t"
      "fma.rn.f32x2 a, w, x, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(w), "f"(x0), "f"(x1));
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

template <typename O, int NV>
__device__ __forceinline__ void store_out(O* dst, const float* v);
template <>
__device__ __forceinline__ void store_out<float, 4>(float* dst, const float* v) {
  *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store_out<float, 8>(float* dst, const float* v) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16, 8>(__nv_bfloat16* dst, const float* v) {
  *reinterpret_cast<uint4*>(dst) =
      make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16, 4>(__nv_bfloat16* dst, const float* v) {
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
}

// The bag's token from its fp32 accumulation (this lane's CI x NV columns, column
// (c * LPR + lane) * NV + i) and its weight sum: the mean divides by the weight sum (zero
// when it is zero), the sum keeps the accumulation, the max gives zero for a bag without
// rows; then the optional LayerNorm over the D columns that the LPR lanes of the group
// hold.  Every lane of the warp calls it (the LayerNorm reductions are shuffles).
template <int LPR, int CI, int NV>
__device__ __forceinline__ void finish_bag(float (&r)[CI][NV], const float (&acc)[CI][NV], float wsum,
                                           bool bad_table, int agg, bool is_max, bool post_ln) {
  constexpr int D = LPR * CI * NV;
  // the mean multiplies by one correctly rounded reciprocal of the weight sum (one IEEE
  // divide per bag, not per column); scaling every weight by 2^k scales the sum and the
  // reciprocal exactly, so the token stays bit-identical
  const float inv = wsum != 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int c = 0; c < CI; ++c)
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float a = acc[c][i];
      r[c][i] = bad_table                ? 0.f
                : agg == TR_AGG_MEAN     ? a * inv
                : is_max                 ? (a == -INFINITY ? 0.f : a)
                                         : a;
    }
  if (post_ln) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) s += r[c][i];
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mean = s * (1.f / D);
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) q = fmaf(r[c][i] - mean, r[c][i] - mean, q);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
    const float rstd = rsqrtf(q * (1.f / D) + kLnEps);
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) r[c][i] = (r[c][i] - mean) * rstd;
  }
}

// Up to UNROLL rows of one chunk of LPR keys into the group's accumulator: the keys and
// weights sit one per lane of the group (k < 0 for none), rows j0 .. j0 + UNROLL - 1 of the
// chunk are loaded before any is consumed, and `between()` runs while they are in flight.
// cnt: the group's keys in this chunk.
template <typename T, int LPR, int CI, int UNROLL, typename Between>
__device__ __forceinline__ void gather_rows(float (&acc)[CI][Vec16<T>::N], const T* table, int k, float v, int cnt,
                                            int j0, int cl, bool is_max, Between&& between) {
  constexpr int NV = Vec16<T>::N;
  constexpr int D = LPR * CI * NV;
  uint4 raw[UNROLL][CI];
  float wv[UNROLL];
  bool lv[UNROLL];
#pragma unroll
  for (int u = 0; u < UNROLL; ++u) {
    const int j = j0 + u;
    const int kk = __shfl_sync(0xffffffffu, k, j % LPR, LPR);
    wv[u] = __shfl_sync(0xffffffffu, v, j % LPR, LPR);
    const bool live = j < cnt && kk >= 0;
    lv[u] = live;
    if (!live) wv[u] = 0.f;
    const uint4* row = reinterpret_cast<const uint4*>(table + (int64_t)(live ? kk : 0) * D);
#pragma unroll
    for (int c = 0; c < CI; ++c) raw[u][c] = live ? ld_stream(row + c * LPR + cl) : make_uint4(0, 0, 0, 0);
  }
  between();
  if (is_max) {
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
#pragma unroll
      for (int c = 0; c < CI; ++c) {
        float f[NV];
        Vec16<T>::unpack(raw[u][c], f);
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[c][i] = lv[u] ? fmaxf(acc[c][i], f[i]) : acc[c][i];
      }
  } else {
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
#pragma unroll
      for (int c = 0; c < CI; ++c) {
        float f[NV];
        Vec16<T>::unpack(raw[u][c], f);
#pragma unroll
        for (int i = 0; i < NV; i += 2) fma2(acc[c][i], acc[c][i + 1], wv[u], f[i], f[i + 1]);
      }
  }
}

// LPR lanes per row, CI 16-byte column blocks per lane (D = LPR * CI * NV).
//
// Each group of LPR lanes owns one bag at a time (a warp works on 32 / LPR bags at once)
// and keeps up to UNROLL row loads in flight, so a warp has several bags' rows in flight
// and needs no cross-lane reduction of the row sums.  A bag costs three dependent memory
// round trips (table id and offsets -> keys and weights -> rows); the group hides two of
// them behind the previous bag: the next bag's table id and offsets are requested when a
// bag starts, and its first LPR keys and weights once the current rows are in flight.
// Loop trip counts are the warp's maximum, so every shuffle is warp-uniform.
// VAR = false compiles the plain weighted average (TR_AGG_MEAN without LayerNorm) only;
// VAR = true reads the aggregator and the LayerNorm flag from `mode`.
template <typename T, typename O, int LPR, int CI, bool VAR, int MINB>
__global__ void __launch_bounds__(256, MINB) wavg_kernel(TableSet tabs, int n_tables,
                                                      const int32_t* __restrict__ bag_table,
                                                      const int64_t* __restrict__ offsets,
                                                      const int32_t* __restrict__ keys,
                                                      const float* __restrict__ weights, int64_t n_bags,
                                                      int mode, O* __restrict__ out, int* status) {
  constexpr int NV = Vec16<T>::N;
  constexpr int D = LPR * CI * NV;
  constexpr int G = 32 / LPR;                 // bags per warp
  constexpr int UNROLL = LPR < 8 ? LPR : 8;   // rows in flight per lane group
  const int lane = threadIdx.x & 31;
  const int grp = lane / LPR;
  const int cl = lane % LPR;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x >> 5) * G;
  const int agg = VAR ? mode & 0xFF : TR_AGG_MEAN;   // TR_AGG_MEAN / TR_AGG_SUM / TR_AGG_MAX
  const bool is_max = VAR && agg == TR_AGG_MAX, post_ln = VAR && (mode & TR_AGG_POST_LN) != 0;
  bool bad = false;

  // the first bag's header and first key chunk
  int tbl_n = 0;
  int64_t s0_n = 0, s1_n = 0;
  int k_n = -1;
  float v_n = 0.f;
  {
    const int64_t b = warp * G + grp;
    if (b < n_bags) {
      tbl_n = __ldg(bag_table + b);
      s0_n = __ldg(offsets + b);
      s1_n = __ldg(offsets + b + 1);
      if (cl < s1_n - s0_n) {
        k_n = __ldg(keys + s0_n + cl);
        v_n = __ldg(weights + s0_n + cl);
      }
    }
  }
  for (int64_t it = warp * G; it < n_bags; it += stride) {
    const int64_t b = it + grp;
    const bool live_bag = b < n_bags;
    const int tbl = tbl_n;
    const int64_t s0 = s0_n, s1 = s1_n;
    int k = k_n;
    float v = v_n;
    const int64_t b2 = b + stride;
    const bool has_next = b2 < n_bags;
    if (has_next) {
      tbl_n = __ldg(bag_table + b2);
      s0_n = __ldg(offsets + b2);
      s1_n = __ldg(offsets + b2 + 1);
    }
    bool next_keys = false;   // the next bag's first key chunk requested yet
    auto fetch_next_keys = [&]() {
      next_keys = true;
      k_n = -1;
      v_n = 0.f;
      if (cl < s1_n - s0_n) {
        k_n = __ldg(keys + s0_n + cl);
        v_n = __ldg(weights + s0_n + cl);
      }
    };
    const bool bad_table = live_bag && (tbl < 0 || tbl >= n_tables);
    bad |= bad_table;
    const int n = (live_bag && !bad_table) ? (int)(s1 - s0) : 0;
    const int n_max = __reduce_max_sync(0xffffffffu, n);   // the warp's longest bag
    const T* table = static_cast<const T*>(tabs.ptr[n > 0 ? tbl : 0]);
    const int64_t nrows = n > 0 ? tabs.rows[tbl] : 0;
    float acc[CI][NV];
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[c][i] = is_max ? -INFINITY : 0.f;
    float wsum = 0.f;
    for (int base = 0; base < n_max; base += LPR) {
      const int cnt = n - base;                     // keys of this bag in the chunk (may be <= 0)
      if (base != 0) {                              // chunks after the prefetched one
        k = -1;
        v = 0.f;
        if (cl < cnt) {
          k = __ldg(keys + s0 + base + cl);
          v = __ldg(weights + s0 + base + cl);
        }
      }
      if (cl >= cnt) {
        k = -1;
        v = 0.f;
      } else if (k < 0 || (int64_t)k >= nrows) {
        bad = true;
        k = -1;
        v = 0.f;
      }
      wsum += v;
      const int cnt_max = n_max - base < LPR ? n_max - base : LPR;   // warp-uniform
      for (int j0 = 0; j0 < cnt_max; j0 += UNROLL)
        gather_rows<T, LPR, CI, UNROLL>(acc, table, k, v, cnt, j0, cl, is_max, [&]() {
          if (has_next && !next_keys) fetch_next_keys();   // overlaps these rows
        });
    }
    if (has_next && !next_keys) fetch_next_keys();   // empty or rejected bag
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    float r[CI][NV];
    finish_bag<LPR, CI, NV>(r, acc, wsum, bad_table, agg, is_max, post_ln);
    if (live_bag) {
#pragma unroll
      for (int c = 0; c < CI; ++c) store_out<O, NV>(out + b * D + (c * LPR + cl) * NV, r[c]);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, STATUS_KEY_RANGE);
}

// Few bags: one block (256 threads) per bag, grid-stride over bags.  The block's
// NG = 256 / LPR lane groups share the bag: group g takes entries g, g + NG, g + 2 NG, ...
// (each lane of a group fetches one key and weight of the group's next LPR entries, so a
// chunk of the block reads NG * LPR = 256 consecutive entries), gathers their rows with
// up to UNROLL in flight, and leaves its partial sum (or max) and weight sum in shared
// memory.  Warp 0 combines the NG partials in group order and finishes the bag as
// wavg_kernel does.  A bag of n rows takes about n / (NG * UNROLL) rounds of row loads
// instead of n / UNROLL.
template <typename T, typename O, int LPR, int CI, bool VAR>
__global__ void __launch_bounds__(256, 4) wavg_split_kernel(TableSet tabs, int n_tables,
                                                            const int32_t* __restrict__ bag_table,
                                                            const int64_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ keys,
                                                            const float* __restrict__ weights, int64_t n_bags,
                                                            int mode, O* __restrict__ out, int* status) {
  constexpr int NV = Vec16<T>::N;
  constexpr int D = LPR * CI * NV;
  constexpr int NG = 256 / LPR;
  constexpr int UNROLL = LPR < 8 ? LPR : 8;
  __shared__ float part[NG][D];               // 256 * CI * NV floats: at most 32 KB
  __shared__ float part_w[NG];
  const int lane = threadIdx.x & 31;
  const int grp = threadIdx.x / LPR;
  const int cl = threadIdx.x % LPR;
  const int agg = VAR ? mode & 0xFF : TR_AGG_MEAN;
  const bool is_max = VAR && agg == TR_AGG_MAX, post_ln = VAR && (mode & TR_AGG_POST_LN) != 0;
  bool bad = false;
  for (int64_t b = blockIdx.x; b < n_bags; b += gridDim.x) {   // block-uniform
    const int tbl = __ldg(bag_table + b);
    const int64_t s0 = __ldg(offsets + b), s1 = __ldg(offsets + b + 1);
    const bool bad_table = tbl < 0 || tbl >= n_tables;
    bad |= bad_table;
    const int n = bad_table ? 0 : (int)(s1 - s0);
    const int mine = n > grp ? (n - grp + NG - 1) / NG : 0;          // this group's entries
    const int mine_max = __reduce_max_sync(0xffffffffu, mine);
    const T* table = static_cast<const T*>(tabs.ptr[n > 0 ? tbl : 0]);
    const int64_t nrows = n > 0 ? tabs.rows[tbl] : 0;
    float acc[CI][NV];
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[c][i] = is_max ? -INFINITY : 0.f;
    float wsum = 0.f;
    for (int base = 0; base < mine_max; base += LPR) {
      const int cnt = mine - base;
      int k = -1;
      float v = 0.f;
      if (cl < cnt) {
        const int64_t e = s0 + grp + (int64_t)NG * (base + cl);
        k = __ldg(keys + e);
        v = __ldg(weights + e);
        if (k < 0 || (int64_t)k >= nrows) {
          bad = true;
          k = -1;
          v = 0.f;
        }
      }
      wsum += v;
      const int cnt_max = mine_max - base < LPR ? mine_max - base : LPR;   // warp-uniform
      for (int j0 = 0; j0 < cnt_max; j0 += UNROLL)
        gather_rows<T, LPR, CI, UNROLL>(acc, table, k, v, cnt, j0, cl, is_max, []() {});
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) part[grp][(c * LPR + cl) * NV + i] = acc[c][i];
    if (cl == 0) part_w[grp] = wsum;
    __syncthreads();
    if (threadIdx.x < 32) {   // warp 0: every group in it combines the same columns; group 0 stores
      float tot[CI][NV];
#pragma unroll
      for (int c = 0; c < CI; ++c)
#pragma unroll
        for (int i = 0; i < NV; ++i) tot[c][i] = is_max ? -INFINITY : 0.f;
      float ws = 0.f;
      for (int g = 0; g < NG; ++g) {
#pragma unroll
        for (int c = 0; c < CI; ++c)
#pragma unroll
          for (int i = 0; i < NV; ++i) {
            const float x = part[g][(c * LPR + cl) * NV + i];
            tot[c][i] = is_max ? fmaxf(tot[c][i], x) : tot[c][i] + x;
          }
        ws += part_w[g];
      }
      float r[CI][NV];
      finish_bag<LPR, CI, NV>(r, tot, ws, bad_table, agg, is_max, post_ln);
      if (grp == 0) {
#pragma unroll
        for (int c = 0; c < CI; ++c) store_out<O, NV>(out + b * D + (c * LPR + cl) * NV, r[c]);
      }
    }
    __syncthreads();          // the partials are rewritten by the next bag
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, STATUS_KEY_RANGE);
}

template <typename T, typename O>
tr_status dispatch(const TableSet& ts, int n_tables, const int32_t* bag_table, const int64_t* offsets,
                   const int32_t* keys, const float* weights, int64_t n_bags, int D, int mode, O* out,
                   int* status, cudaStream_t st) {
  constexpr int NV = Vec16<T>::N;
  const int vecs = D / NV;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 8 warps per block, 32 / LPR bags per warp at a time.  With one 16-byte vector per lane
  // (CI = 1) 4 blocks per SM are resident and the grid is 32 blocks per SM, so that blocks
  // started late (an SM held by a concurrent kernel) take a small share of the work.  Rows
  // of 16 vectors (a 256-byte bf16 row of D = 128) go to 8 lanes with two vectors each: half
  // the lanes per row and twice the bags per warp halve the per-bag instructions of the
  // group (headers, key chunks, the weight-sum reduction and the finish); that needs more
  // registers, so 2 blocks per SM are resident and the grid is 16 blocks per SM.
  auto grid_of = [&](int lpr, int per_sm) {
    const int64_t bags_per_block = 8 * (32 / lpr);
    const int64_t blocks_needed = (n_bags + bags_per_block - 1) / bags_per_block;
    return (int)std::max<int64_t>(1, std::min<int64_t>(blocks_needed, (int64_t)sms * per_sm));
  };
  // few bags (one resident round of one-bag blocks, 4 per SM): a block per bag
  const bool split = n_bags <= (int64_t)sms * 4;
  const int grid_split = (int)std::max<int64_t>(1, n_bags);
#define TR_WAVG_K(K, G, LPR, CI, VAR, ...) \
  K<T, O, LPR, CI, VAR, ##__VA_ARGS__><<<G, 256, 0, st>>>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, mode, out, status)
#define TR_WAVG(LPR, CI, MINB, PER_SM, SLPR, SCI)                                                     \
  if (split && mode == TR_AGG_MEAN) TR_WAVG_K(wavg_split_kernel, grid_split, SLPR, SCI, false);            \
  else if (split) TR_WAVG_K(wavg_split_kernel, grid_split, SLPR, SCI, true);                               \
  else if (mode == TR_AGG_MEAN) TR_WAVG_K(wavg_kernel, grid_of(LPR, PER_SM), LPR, CI, false, MINB);        \
  else TR_WAVG_K(wavg_kernel, grid_of(LPR, PER_SM), LPR, CI, true, MINB)
  // (the block-per-bag kernel keeps one vector per lane and 16-lane groups)
  switch (vecs) {
    case 1: TR_WAVG(1, 1, 4, 32, 1, 1); break;
    case 2: TR_WAVG(2, 1, 4, 32, 2, 1); break;
    case 4: TR_WAVG(4, 1, 4, 32, 4, 1); break;
    case 8: TR_WAVG(8, 1, 4, 32, 8, 1); break;
    case 16: TR_WAVG(8, 2, 2, 16, 16, 1); break;
    case 32: TR_WAVG(32, 1, 4, 32, 32, 1); break;
    case 64: TR_WAVG(32, 2, 4, 32, 32, 2); break;
    case 128: TR_WAVG(32, 4, 4, 32, 32, 4); break;
    default: return fail(TR_ERR_UNSUPPORTED, "tr_aggregate: D=%d gives %d vectors per row (need 1..32 as a power of two, 64 or 128)", D, vecs);
  }
#undef TR_WAVG
#undef TR_WAVG_K
  TR_LAUNCH_CHECK(split ? "wavg_split_kernel" : "wavg_kernel");
  return TR_OK;
}

}  // namespace

tr_status launch_aggregate(const tr_table* tables, int n_tables, const int32_t* bag_table,
                           const int64_t* offsets, const int32_t* keys, const float* weights,
                           int64_t n_bags, int D, tr_dtype out_dtype, int mode, void* out, cudaStream_t st) {
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  TableSet ts = {};
  for (int i = 0; i < n_tables; ++i) {
    ts.ptr[i] = tables[i].data;
    ts.rows[i] = tables[i].n_rows;
  }
  const tr_dtype tdt = tables[0].dtype;
  if (tdt == TR_BF16 && out_dtype == TR_BF16)
    return dispatch<__nv_bfloat16, __nv_bfloat16>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D, mode,
                                                  static_cast<__nv_bfloat16*>(out), ds->status, st);
  if (tdt == TR_BF16 && out_dtype == TR_F32)
    return dispatch<__nv_bfloat16, float>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D, mode,
                                          static_cast<float*>(out), ds->status, st);
  if (tdt == TR_F32 && out_dtype == TR_F32)
    return dispatch<float, float>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D, mode,
                                  static_cast<float*>(out), ds->status, st);
  return dispatch<float, __nv_bfloat16>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D, mode,
                                        static_cast<__nv_bfloat16*>(out), ds->status, st);
}

}  // namespace tr
