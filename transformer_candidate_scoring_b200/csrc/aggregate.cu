// Weighted-average aggregation of (key, weight) bags (TransRetrieval §3.2):
//   out[b] = sum_i v_i h(k_i) / sum_i v_i
//
// HBM-bound gather.  One warp owns one bag at a time (grid-stride over bags).  A table
// row is split into 16-byte vectors; `LPR` lanes cover one row, so a warp reads
// 32/LPR rows per step (two 256-byte rows for D = 128 bf16).  Keys and weights of up to
// 32 entries are fetched with one coalesced load each and broadcast by shuffle; row
// loads of four steps are issued before any is consumed, so each lane keeps several
// 16-byte reads in flight.  Accumulation is fp32; the division by the weight sum is a
// correctly rounded IEEE divide, so scaling all weights of a bag by 2^k leaves the
// result bit-identical.
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

// LPR lanes per row, CI 16-byte column blocks per lane (D = LPR * CI * NV).
template <typename T, typename O, int LPR, int CI>
__global__ void __launch_bounds__(256) wavg_kernel(TableSet tabs, int n_tables,
                                                   const int32_t* __restrict__ bag_table,
                                                   const int64_t* __restrict__ offsets,
                                                   const int32_t* __restrict__ keys,
                                                   const float* __restrict__ weights, int64_t n_bags,
                                                   O* __restrict__ out, int* status) {
  constexpr int NV = Vec16<T>::N;
  constexpr int D = LPR * CI * NV;
  constexpr int RPS = 32 / LPR;   // rows per warp step
  constexpr int UNROLL = 4;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR;
  const int cl = lane % LPR;
  const int64_t warp = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);

  for (int64_t b = warp; b < n_bags; b += nwarps) {
    const int tbl = __ldg(bag_table + b);
    const int64_t s0 = __ldg(offsets + b), s1 = __ldg(offsets + b + 1);
    float acc[CI][NV];
#pragma unroll
    for (int c = 0; c < CI; ++c)
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[c][i] = 0.f;
    float wsum = 0.f;
    bool bad = false;
    if (tbl < 0 || tbl >= n_tables) {
      bad = true;
    } else {
      const T* table = static_cast<const T*>(tabs.ptr[tbl]);
      const int64_t nrows = tabs.rows[tbl];
      for (int64_t base = s0; base < s1; base += 32) {
        const int cnt = (int)(s1 - base < 32 ? s1 - base : 32);
        int k = -1;
        float v = 0.f;
        if (lane < cnt) {
          k = __ldg(keys + base + lane);
          v = __ldg(weights + base + lane);
          if (k < 0 || (int64_t)k >= nrows) {
            bad = true;
            k = -1;
            v = 0.f;
          }
        }
        wsum += v;
        for (int j0 = 0; j0 < cnt; j0 += RPS * UNROLL) {
          uint4 raw[UNROLL][CI];
          float wv[UNROLL];
#pragma unroll
          for (int u = 0; u < UNROLL; ++u) {
            const int j = j0 + u * RPS + sub;
            const int kk = __shfl_sync(0xffffffffu, k, j & 31);
            wv[u] = __shfl_sync(0xffffffffu, v, j & 31);
            const bool live = (j < cnt) && kk >= 0;
            if (!live) wv[u] = 0.f;
            const uint4* row = reinterpret_cast<const uint4*>(table + (int64_t)(live ? kk : 0) * D);
#pragma unroll
            for (int c = 0; c < CI; ++c)
              raw[u][c] = live ? ld_stream(row + c * LPR + cl) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int u = 0; u < UNROLL; ++u)
#pragma unroll
            for (int c = 0; c < CI; ++c) {
              float f[NV];
              Vec16<T>::unpack(raw[u][c], f);
#pragma unroll
              for (int i = 0; i < NV; ++i) acc[c][i] = fmaf(wv[u], f[i], acc[c][i]);
            }
        }
      }
    }
    // combine the RPS row-groups and the weight sum across the warp
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
      for (int c = 0; c < CI; ++c)
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[c][i] += __shfl_xor_sync(0xffffffffu, acc[c][i], off);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, STATUS_KEY_RANGE);
    const bool bad_table = (tbl < 0 || tbl >= n_tables);
    if (sub == 0) {
#pragma unroll
      for (int c = 0; c < CI; ++c) {
        float r[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) r[i] = (wsum != 0.f && !bad_table) ? acc[c][i] / wsum : 0.f;
        store_out<O, NV>(out + b * D + (c * LPR + cl) * NV, r);
      }
    }
  }
}

template <typename T, typename O>
tr_status dispatch(const TableSet& ts, int n_tables, const int32_t* bag_table, const int64_t* offsets,
                   const int32_t* keys, const float* weights, int64_t n_bags, int D, O* out, int* status,
                   cudaStream_t st) {
  constexpr int NV = Vec16<T>::N;
  const int vecs = D / NV;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t blocks_needed = (n_bags + 7) / 8;
  const int grid = (int)std::min<int64_t>(blocks_needed, (int64_t)sms * 8);
#define TR_WAVG(LPR, CI)                                                                               \
  wavg_kernel<T, O, LPR, CI><<<grid, 256, 0, st>>>(ts, n_tables, bag_table, offsets, keys, weights, \
                                                   n_bags, out, status)
  switch (vecs) {
    case 1: TR_WAVG(1, 1); break;
    case 2: TR_WAVG(2, 1); break;
    case 4: TR_WAVG(4, 1); break;
    case 8: TR_WAVG(8, 1); break;
    case 16: TR_WAVG(16, 1); break;
    case 32: TR_WAVG(32, 1); break;
    case 64: TR_WAVG(32, 2); break;
    case 128: TR_WAVG(32, 4); break;
    default: return fail(TR_ERR_UNSUPPORTED, "tr_aggregate: D=%d gives %d vectors per row (need 1..32 as a power of two, 64 or 128)", D, vecs);
  }
#undef TR_WAVG
  TR_LAUNCH_CHECK("wavg_kernel");
  return TR_OK;
}

}  // namespace

tr_status launch_aggregate(const tr_table* tables, int n_tables, const int32_t* bag_table,
                           const int64_t* offsets, const int32_t* keys, const float* weights,
                           int64_t n_bags, int D, tr_dtype out_dtype, void* out, cudaStream_t st) {
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  TableSet ts = {};
  for (int i = 0; i < n_tables; ++i) {
    ts.ptr[i] = tables[i].data;
    ts.rows[i] = tables[i].n_rows;
  }
  const tr_dtype tdt = tables[0].dtype;
  if (tdt == TR_BF16 && out_dtype == TR_BF16)
    return dispatch<__nv_bfloat16, __nv_bfloat16>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D,
                                                  static_cast<__nv_bfloat16*>(out), ds->status, st);
  if (tdt == TR_BF16 && out_dtype == TR_F32)
    return dispatch<__nv_bfloat16, float>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D,
                                          static_cast<float*>(out), ds->status, st);
  if (tdt == TR_F32 && out_dtype == TR_F32)
    return dispatch<float, float>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D,
                                  static_cast<float*>(out), ds->status, st);
  return dispatch<float, __nv_bfloat16>(ts, n_tables, bag_table, offsets, keys, weights, n_bags, D,
                                        static_cast<__nv_bfloat16*>(out), ds->status, st);
}

}  // namespace tr
