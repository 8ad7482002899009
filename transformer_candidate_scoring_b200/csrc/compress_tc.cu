// Target compressor on tcgen05 tensor cores (TransRetrieval §3.3):
//   t = W3 g2(W2 g1(W1 x + b1) + b2) + b3,   g_i(z) = LayerNorm_i(PReLU_i(z))
//
// One persistent CTA per SM walks 128-row tiles and keeps each tile on chip through all
// three layers:
//   layer 1: x tiles arrive by TMA tensor loads (128-byte swizzle, rows past the end are
//            zero-filled by the copy engine) together with bulk copies of the matching
//            W1 slice, two stages deep; the [128 x c1] fp32 accumulator fills TMEM.
//   epilogue 1: + b1, PReLU, LayerNorm over c1 (two passes over TMEM), fp16 result written
//            in the core-matrix layout over the now idle stage buffers.
//   layers 2, 3: W2 / W3 slices (fp16) stream through a second two-stage ring; the hidden
//            activations and these weights are fp16 operands (x and W1 stay bf16, x's
//            storage type), which rounds them 8x more finely than bf16 at the same rate.
//   epilogue 3: + b3, fp32 tokens straight to global memory.
// Warp 0 issues copies, warp 1 issues MMAs, warps 2-9 run the epilogues: two warps per TMEM
// lane quadrant, each owning half of a row's columns; a row's LayerNorm statistics are merged
// across the pair (Welford) through shared memory.  Waits are bounded as in the candidate
// stack kernel.  Every tile is claimed at run time from a per-launch counter: a CTA that
// starts late, on an SM another kernel still holds, finds less work (or none) instead of
// holding the launch back.  The producer passes each claimed tile index to the MMA and
// epilogue threads through a two-entry ring in shared memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "model.cuh"
#include "tc_common.cuh"

namespace tr {
namespace {

using namespace tc;

constexpr int kM = 128;
constexpr int STAGE1 = 80 * 1024;              // x slice (16 KB) + W1 slice (<= 64 KB)
constexpr int OFF_R1 = 0;
constexpr int OFF_R2 = 2 * STAGE1;             // 160 KB
constexpr int STAGE2 = 32 * 1024;
constexpr int OFF_BAR = OFF_R2 + 2 * STAGE2;   // 224 KB
constexpr int OFF_B3 = OFF_BAR + 256;           // the last layer's bias (c3 <= 256 floats)
constexpr int SMEM_BYTES = OFF_B3 + 1024 + 1024;
// The per-column vectors of the layer whose epilogue runs are staged in shared memory at
// R1 + 132 KB (8 KB): that part of the second x/W1 stage is idle from the end of a tile's
// first GEMM until the next tile's loads, which wait for its last GEMM.
constexpr int OFF_VEC = OFF_R1 + 132 * 1024;

struct CompParams {
  CUtensorMap xmap;            // x [n][c0] bf16, box {64, 128}, 128-byte swizzle
  const uint8_t* w1;           // [c0/64] slices of W1^T [c1 x 64]
  const uint8_t* w2;           // [c1/64] slices of W2^T [c2 x 64]
  const uint8_t* w3;           // [c2/64] slices of W3^T [c3 x 64]
  const float* vec;            // b1 a1 g1 be1 (c1 each), b2 a2 g2 be2 (c2 each), b3 (c3)
  float* out;                  // [n][c3]
  int* status;
  int* claim;                  // next unclaimed tile (zero at launch)
  long long n;
  int n_tiles, c0, c1, c2, c3;
};

struct CBars {
  uint32_t full1[2], empty1[2], full2[2], empty2[2], r1_free, mma, epi, drain, qsync[4], vsync;
  uint32_t tile_full[2], tile_empty[2], tile_slot[2];   // the claimed-tile ring
};

// Next tile index of this CTA from the two-entry ring (-1: no more); the reader releases
// the entry at once.
__device__ __forceinline__ int next_tile(const CBars& b, int& ts, uint32_t& tph, volatile int* abort_flag,
                                         bool& ok) {
  ok = ok && mbar_wait(b.tile_full[ts], tph, abort_flag);
  int t = -1;
  if (ok) asm volatile("ld.shared.b32 %0, [%1];" : "=r"(t) : "r"(b.tile_slot[ts]) : "memory");
  mbar_arrive(b.tile_empty[ts]);
  if (++ts == 2) {
    ts = 0;
    tph ^= 1;
  }
  return ok ? t : -1;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// fp16 x fp16 -> fp32, both operands K-major
constexpr uint32_t idesc_f16c(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_h2c(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// K-major operand written by TMA with the 128-byte swizzle: 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
}

__device__ void comp_producer(const CompParams& p, uint32_t r1, uint32_t r2, const CBars& b, volatile int* abort_flag) {
  int s1 = 0, s2 = 0;
  uint32_t ph1 = 0, ph2 = 0, free_phase = 0;
  const uint32_t w1_bytes = p.c1 * 128, w2_bytes = p.c2 * 128, w3_bytes = p.c3 * 128;
  bool ok = true;
  bool pend1[2] = {false, false}, pend2[2] = {false, false};
  uint32_t par1[2] = {0, 0}, par2[2] = {0, 0};
  int ts = 0;
  uint32_t tph = 0;
  for (int tile = atomicAdd(p.claim, 1); ok;) {
    // publish the tile (or the end) to the MMA and epilogue threads
    if (!(ok = mbar_wait(b.tile_empty[ts], tph ^ 1, abort_flag))) break;
    const int pub = tile < p.n_tiles ? tile : -1;
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(b.tile_slot[ts]), "r"(pub) : "memory");
    mbar_arrive(b.tile_full[ts]);
    if (++ts == 2) {
      ts = 0;
      tph ^= 1;
    }
    if (pub < 0) break;
    // the stage buffers hold the previous tile's activations until its last GEMM is done
    if (!(ok = mbar_wait(b.r1_free, free_phase ^ 1, abort_flag))) break;
    free_phase ^= 1;
    for (int kc = 0; kc < p.c0 / 64 && ok; ++kc) {
      if (!(ok = mbar_wait(b.empty1[s1], ph1 ^ 1, abort_flag))) break;
      const uint32_t st = r1 + s1 * STAGE1;
      mbar_arrive_expect_tx(b.full1[s1], kM * 64 * 2 + w1_bytes);
      tma_load_2d(st, &p.xmap, kc * 64, tile * kM, b.full1[s1]);
      bulk_g2s(st + 16384, p.w1 + (size_t)kc * w1_bytes, w1_bytes, b.full1[s1]);
      pend1[s1] = true;
      par1[s1] = ph1;
      if (++s1 == 2) { s1 = 0; ph1 ^= 1; }
    }
    for (int j = 0; j < p.c1 / 64 + p.c2 / 64 && ok; ++j) {
      if (!(ok = mbar_wait(b.empty2[s2], ph2 ^ 1, abort_flag))) break;
      const bool is2 = j < p.c1 / 64;
      const uint32_t bytes = is2 ? w2_bytes : w3_bytes;
      const uint8_t* src = is2 ? p.w2 + (size_t)j * w2_bytes : p.w3 + (size_t)(j - p.c1 / 64) * w3_bytes;
      mbar_arrive_expect_tx(b.full2[s2], bytes);
      bulk_g2s(r2 + s2 * STAGE2, src, bytes, b.full2[s2]);
      pend2[s2] = true;
      par2[s2] = ph2;
      if (++s2 == 2) { s2 = 0; ph2 ^= 1; }
    }
    tile = atomicAdd(p.claim, 1);
  }
  if (!ok) {
    for (int s = 0; s < 2; ++s) {
      for (uint64_t t0 = globaltimer_ns(); pend1[s] && !mbar_try_wait(b.full1[s], par1[s]) && globaltimer_ns() - t0 < 200000000ull;) {
      }
      for (uint64_t t0 = globaltimer_ns(); pend2[s] && !mbar_try_wait(b.full2[s], par2[s]) && globaltimer_ns() - t0 < 200000000ull;) {
      }
    }
  }
}

__device__ void comp_mma(const CompParams& p, uint32_t tmem, uint32_t r1, uint32_t r2, const CBars& b,
                         volatile int* abort_flag) {
  int s1 = 0, s2 = 0;
  uint32_t ph1 = 0, ph2 = 0, epi_phase = 0;
  bool ok = true;
  const int n1 = std::min(p.c1, 256);
  // layer 1 multiplies bf16 x by bf16 W1; layers 2 and 3 fp16 activations by fp16 weights
  const uint32_t id1 = idesc_bf16(kM, n1), id2 = idesc_f16c(kM, p.c2), id3 = idesc_f16c(kM, p.c3);
  auto wait_epi = [&]() {
    ok = ok && mbar_wait(b.epi, epi_phase, abort_flag);
    epi_phase ^= 1;
    tc_fence_after();
    return ok;
  };
  int ts = 0;
  uint32_t tph = 0;
  for (bool first = true; ok; first = false) {
    const int tile = next_tile(b, ts, tph, abort_flag, ok);
    if (tile < 0) break;
    if (!first && !wait_epi()) break;   // previous tile's last epilogue has read TMEM
    // layer 1: [128 x c0] x [c0 x c1]
    for (int kc = 0; kc < p.c0 / 64 && ok; ++kc) {
      if (!(ok = mbar_wait(b.full1[s1], ph1, abort_flag))) break;
      tc_fence_after();
      const uint32_t xa = r1 + s1 * STAGE1, wb = xa + 16384;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        for (int nh = 0; nh < p.c1 / n1; ++nh)
          mma_bf16(tmem + nh * n1, sdesc_sw128(xa + kk * 32),
                   sdesc(wb + kk * 2 * p.c1 * 16 + nh * (n1 / 8) * 128, p.c1 * 16, 128), id1,
                   (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(b.empty1[s1]);
      if (++s1 == 2) { s1 = 0; ph1 ^= 1; }
    }
    if (!ok) break;
    mma_commit(b.mma);
    if (!wait_epi()) break;                                // h1 (bf16) in R1
    for (int kc = 0; kc < p.c1 / 64 && ok; ++kc) {
      if (!(ok = mbar_wait(b.full2[s2], ph2, abort_flag))) break;
      tc_fence_after();
      const uint32_t wb = r2 + s2 * STAGE2;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem, sdesc(r1 + (4 * kc + kk) * 2 * kM * 16, kM * 16, 128),
                 sdesc(wb + kk * 2 * p.c2 * 16, p.c2 * 16, 128), id2, (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(b.empty2[s2]);
      if (++s2 == 2) { s2 = 0; ph2 ^= 1; }
    }
    if (!ok) break;
    mma_commit(b.mma);
    if (!wait_epi()) break;                                // h2 (bf16) in R1
    for (int kc = 0; kc < p.c2 / 64 && ok; ++kc) {
      if (!(ok = mbar_wait(b.full2[s2], ph2, abort_flag))) break;
      tc_fence_after();
      const uint32_t wb = r2 + s2 * STAGE2;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16(tmem + 256, sdesc(r1 + (4 * kc + kk) * 2 * kM * 16, kM * 16, 128),
                 sdesc(wb + kk * 2 * p.c3 * 16, p.c3 * 16, 128), id3, (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(b.empty2[s2]);
      if (++s2 == 2) { s2 = 0; ph2 ^= 1; }
    }
    if (!ok) break;
    mma_commit(b.r1_free);
    mma_commit(b.mma);
  }
  mma_commit(b.drain);
  for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.drain, 0) && globaltimer_ns() - t0 < 500000000ull;) {
  }
}

// Epilogue threads: two warps per TMEM lane quadrant, each owning half of a row's columns.
struct CEpi {
  uint32_t trow, rowoff, xbuf;
  int m, hf, q;
  uint32_t qbar;
  uint32_t ph_q;
  volatile int* abort_flag;
  bool ok;
  // exchange one float2 with the other half of this row (slot alternates between uses)
  __device__ float2 swap(float2 mine, int slot) {
    const uint32_t x = xbuf + slot * (2 * kM * 8);
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(x + (hf * kM + m) * 8), "f"(mine.x), "f"(mine.y)
                 : "memory");
    mbar_arrive(qbar);
    ok = ok && mbar_wait(qbar, ph_q, abort_flag);
    ph_q ^= 1;
    float2 o;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(o.x), "=f"(o.y) : "r"(x + ((1 - hf) * kM + m) * 8)
                 : "memory");
    return o;
  }
};

// eight consecutive floats of a vector staged in shared memory
__device__ __forceinline__ void vec8(const float* p, float* o) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

// + bias, PReLU, LayerNorm over the `cols` accumulator columns of this row, of which this
// thread owns [c0, c0 + cols/2); fp16 result into the next layer's operand in R1.
__device__ __forceinline__ void prelu_ln_half(CEpi& e, int cols, const float* bias, const float* slope,
                                              const float* g, const float* be, uint32_t dst_row, int slot) {
  const int half = cols / 2, c0 = e.hf * half;
  const uint32_t tcol = e.trow + c0;
  float x0 = 0.f, s1 = 0.f, s2 = 0.f;
  for (int c = 0; c < half; c += 32) {
    float v[32];
    tmem_ld16(tcol + c, v);
    tmem_ld16(tcol + c + 16, v + 16);
    tmem_wait_ld();
    reg_fence<32>(v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float bb[8], sl[8];
      vec8(bias + c0 + c + 8 * k, bb);
      vec8(slope + c0 + c + 8 * k, sl);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float x = v[8 * k + i] + bb[i];
        x = x >= 0.f ? x : x * sl[i];
        if (c == 0 && k == 0 && i == 0) x0 = x;
        const float d = x - x0;
        s1 += d;
        s2 = fmaf(d, d, s2);
      }
    }
  }
  // this half's mean and sum of squared deviations, merged with the other half (Welford)
  const float inv_h = 1.f / half;
  const float mh = x0 + s1 * inv_h;
  const float m2h = fmaxf(s2 - s1 * s1 * inv_h, 0.f);
  const float2 o = e.swap(make_float2(mh, m2h), slot);
  const float dmu = mh - o.x;
  const float mean = 0.5f * (mh + o.x);
  const float var = (m2h + o.y + dmu * dmu * (0.25f * cols)) / cols;
  const float rstd = rsqrtf(var + kLnEps);
  for (int c = 0; c < half; c += 32) {
    float v[32];
    tmem_ld16(tcol + c, v);
    tmem_ld16(tcol + c + 16, v + 16);
    tmem_wait_ld();
    reg_fence<32>(v);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float bb[8], sl[8], gg[8], ee[8], w[8];
      vec8(bias + c0 + c + 8 * k, bb);
      vec8(slope + c0 + c + 8 * k, sl);
      vec8(g + c0 + c + 8 * k, gg);
      vec8(be + c0 + c + 8 * k, ee);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float x = v[8 * k + i] + bb[i];
        x = x >= 0.f ? x : x * sl[i];
        w[i] = fmaf((x - mean) * rstd, gg[i], ee[i]);
      }
      st_shared_v4(dst_row + ((c0 + c) / 8 + k) * 2048, pack_h2c(w[0], w[1]), pack_h2c(w[2], w[3]),
                   pack_h2c(w[4], w[5]), pack_h2c(w[6], w[7]));
    }
  }
}

__device__ void comp_epilogue(const CompParams& p, uint32_t tmem, uint32_t r1, const CBars& b, float* svec,
                              float* sb3, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  CEpi e;
  e.q = warp & 3;
  e.m = e.q * 32 + lane;
  e.hf = (warp - 2) >> 2;
  e.trow = tmem + ((uint32_t)(e.q * 32) << 16);
  e.rowoff = (e.m >> 3) * 128 + (e.m & 7) * 16;
  e.xbuf = r1 + 128 * 1024;      // idle between the first layer's MMAs and the next tile's loads
  e.qbar = b.qsync[e.q];
  e.ph_q = 0;
  e.abort_flag = abort_flag;
  e.ok = true;
  const float* v1 = p.vec;
  const float* v2 = p.vec + 4 * p.c1;
  const float* b3 = v2 + 4 * p.c2;
  const int et = threadIdx.x - 64;                 // 0 .. 255
  for (int i = et; i < p.c3; i += 256) sb3[i] = __ldg(b3 + i);   // visible after the first vsync
  uint32_t mma_phase = 0, vph = 0;
  // rendezvous of the 256 epilogue threads after a vector staging (bounded)
  auto vbar = [&]() {
    mbar_arrive(b.vsync);
    e.ok = e.ok && mbar_wait(b.vsync, vph, abort_flag);
    vph ^= 1;
    return e.ok;
  };
  auto wait_mma = [&]() {
    e.ok = e.ok && mbar_wait(b.mma, mma_phase, abort_flag);
    mma_phase ^= 1;
    tc_fence_after();
    return e.ok;
  };
  auto signal = [&]() {
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(b.epi);
  };
  int ts = 0;
  uint32_t tph = 0;
  for (;;) {
    const int tile = next_tile(b, ts, tph, abort_flag, e.ok);
    if (tile < 0) break;
    // layer 1's vectors (4 c1 floats) are read into registers while its GEMM runs and
    // stored once it is done
    float4 r1v[2];
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (et + 256 * k < p.c1) r1v[k] = __ldg(reinterpret_cast<const float4*>(v1) + et + 256 * k);
    if (!wait_mma()) break;
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (et + 256 * k < p.c1) reinterpret_cast<float4*>(svec)[et + 256 * k] = r1v[k];
    if (!vbar()) break;
    prelu_ln_half(e, p.c1, svec, svec + p.c1, svec + 2 * p.c1, svec + 3 * p.c1, r1 + e.rowoff, 0);
    signal();
    // layer 2's: every thread has finished reading layer 1's once the layer-2 GEMM is done
    float4 r2v;
    if (et < p.c2) r2v = __ldg(reinterpret_cast<const float4*>(v2) + et);
    if (!wait_mma()) break;
    if (et < p.c2) reinterpret_cast<float4*>(svec)[et] = r2v;
    if (!vbar()) break;
    prelu_ln_half(e, p.c2, svec, svec + p.c2, svec + 2 * p.c2, svec + 3 * p.c2, r1 + e.rowoff, 1);
    signal();
    if (!wait_mma()) break;
    const long long row = (long long)tile * kM + e.m;
    const int h3 = p.c3 / 2;
    for (int c = e.hf * h3; c < (e.hf + 1) * h3; c += 16) {
      float v[16];
      tmem_ld16(e.trow + 256 + c, v);
      tmem_wait_ld();
      reg_fence<16>(v);
      float bb[16];
      vec8(sb3 + c, bb);
      vec8(sb3 + c + 8, bb + 8);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] += bb[i];
      if (row < p.n) {
        float4* dst = reinterpret_cast<float4*>(p.out + row * p.c3 + c);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
    signal();
  }
}

__global__ void __launch_bounds__(320, 1) compress_kernel(const __grid_constant__ CompParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t r1 = base + OFF_R1, r2 = base + OFF_R2, bar0 = base + OFF_BAR;
  CBars b;
  for (int s = 0; s < 2; ++s) {
    b.full1[s] = bar0 + 8 * s;
    b.empty1[s] = bar0 + 16 + 8 * s;
    b.full2[s] = bar0 + 32 + 8 * s;
    b.empty2[s] = bar0 + 48 + 8 * s;
  }
  b.r1_free = bar0 + 64;
  b.mma = bar0 + 72;
  b.epi = bar0 + 80;
  b.drain = bar0 + 88;
  for (int q = 0; q < 4; ++q) b.qsync[q] = bar0 + 96 + 8 * q;
  b.vsync = bar0 + 144;
  for (int s = 0; s < 2; ++s) {
    b.tile_full[s] = bar0 + 152 + 8 * s;
    b.tile_empty[s] = bar0 + 168 + 8 * s;
    b.tile_slot[s] = bar0 + 184 + 4 * s;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + OFF_BAR + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_BAR + 136);
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(b.full1[s], 1);
      mbar_init(b.empty1[s], 1);
      mbar_init(b.full2[s], 1);
      mbar_init(b.empty2[s], 1);
    }
    mbar_init(b.r1_free, 1);
    mbar_init(b.mma, 1);
    mbar_init(b.epi, 256);
    mbar_init(b.drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(b.qsync[q], 64);
    mbar_init(b.vsync, 256);
    for (int s = 0; s < 2; ++s) {
      mbar_init(b.tile_full[s], 1);
      mbar_init(b.tile_empty[s], 1 + 256);   // the MMA thread and every epilogue thread
    }
    *abort_flag = 0;
    mbar_fence_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.xmap)) : "memory");
    // the grid's weight slices (one contiguous image) into L2 at once
    prefetch_l2_share(p.w1, ((size_t)p.c0 * p.c1 + (size_t)p.c1 * p.c2 + (size_t)p.c2 * p.c3) * 2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == 0) {
    if (lane == 0) comp_producer(p, r1, r2, b, abort_flag);
  } else if (warp == 1) {
    if (lane == 0) comp_mma(p, tmem, r1, r2, b, abort_flag);
  } else {
    comp_epilogue(p, tmem, r1, b, reinterpret_cast<float*>(gbase + OFF_VEC), reinterpret_cast<float*>(gbase + OFF_B3),
                  abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, STATUS_KERNEL_TIMEOUT);
}

// W^T slice rows [0, N) x cols [k0, k0 + 64) of W [K][N] in the core-matrix layout, as bf16
// (f16 = false) or fp16.
void put_slice(uint16_t* dst, const float* W, int N, int k0, bool f16) {
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < 64; ++k) {
      float f = W[(size_t)(k0 + k) * N + n];
      uint16_t h;
      if (f16) {
        const __half hv = __float2half_rn(f);
        memcpy(&h, &hv, 2);
      } else {
        uint32_t u;
        memcpy(&u, &f, 4);
        h = (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
      }
      dst[((size_t)(k / 8) * (N / 8) + n / 8) * 64 + (n % 8) * 8 + (k % 8)] = h;
    }
}

// Whether the fp16 operands of layers 2 and 3 stay far inside fp16's range: they are
// LayerNorm outputs (|value| <= max|gain| sqrt(width) + max|shift|) and the weights.
bool comp_fp16_safe(const tr_model_desc& d, const tr_model_weights* w) {
  const int* c = d.comp_dims;
  const double limit = 16384.0;
  for (int i = 0; i < 2; ++i) {
    double g = 0, b = 0, wm = 0;
    for (int j = 0; j < c[i + 1]; ++j) {
      g = std::max(g, (double)fabsf(w->comp_ln_g[i][j]));
      b = std::max(b, (double)fabsf(w->comp_ln_b[i][j]));
    }
    for (size_t j = 0; j < (size_t)c[i + 1] * c[i + 2]; ++j) wm = std::max(wm, (double)fabsf(w->comp_W[i + 1][j]));
    if (!(g * sqrt((double)c[i + 1]) + b < limit && wm < limit)) return false;
  }
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

}  // namespace

bool tc_comp_supported(const tr_model* m) {
  const int* c = m->desc.comp_dims;
  return m->desc.dtype == TR_BF16 && m->tc_comp && c[0] % 64 == 0 && c[1] % 64 == 0 && c[1] <= 512 &&
         c[2] % 64 == 0 && c[2] <= 256 && c[3] % 32 == 0 && c[3] <= 256;
}

// Builds the compressor's weight slices; called from tc_build for bf16 models.
tr_status tc_build_comp(tr_model* m, const tr_model_weights* w) {
  const int* c = m->desc.comp_dims;
  if (!(c[0] % 64 == 0 && c[1] % 64 == 0 && c[1] <= 512 && c[2] % 64 == 0 && c[2] <= 256 && c[3] % 32 == 0 &&
        c[3] <= 256))
    return TR_OK;
  if (!comp_fp16_safe(m->desc, w)) return TR_OK;   // the CUDA-core path serves this model
  const size_t e1 = (size_t)c[0] * c[1], e2 = (size_t)c[1] * c[2], e3 = (size_t)c[2] * c[3];
  std::vector<uint16_t> img(e1 + e2 + e3);
  for (int kc = 0; kc < c[0] / 64; ++kc)
    put_slice(img.data() + (size_t)kc * 64 * c[1], w->comp_W[0], c[1], 64 * kc, false);
  for (int kc = 0; kc < c[1] / 64; ++kc)
    put_slice(img.data() + e1 + (size_t)kc * 64 * c[2], w->comp_W[1], c[2], 64 * kc, true);
  for (int kc = 0; kc < c[2] / 64; ++kc)
    put_slice(img.data() + e1 + e2 + (size_t)kc * 64 * c[3], w->comp_W[2], c[3], 64 * kc, true);
  std::vector<float> vec;
  for (int i = 0; i < 2; ++i) {
    const int n = c[i + 1];
    vec.insert(vec.end(), w->comp_b[i], w->comp_b[i] + n);
    vec.insert(vec.end(), w->comp_prelu[i], w->comp_prelu[i] + n);
    vec.insert(vec.end(), w->comp_ln_g[i], w->comp_ln_g[i] + n);
    vec.insert(vec.end(), w->comp_ln_b[i], w->comp_ln_b[i] + n);
  }
  vec.insert(vec.end(), w->comp_b[2], w->comp_b[2] + c[3]);
  const size_t ib = img.size() * 2, vb = vec.size() * 4;
  void* blob = nullptr;
  if (cudaMalloc(&blob, ib + vb) != cudaSuccess) {
    cudaGetLastError();
    return fail(TR_ERR_NOMEM, "compressor weight images: allocation failed");
  }
  TR_CUDA_TRY(cudaMemcpy(blob, img.data(), ib, cudaMemcpyHostToDevice));
  TR_CUDA_TRY(cudaMemcpy((uint8_t*)blob + ib, vec.data(), vb, cudaMemcpyHostToDevice));
  m->tc_comp = blob;
  m->tc_comp_vec = reinterpret_cast<const float*>((uint8_t*)blob + ib);
  return TR_OK;
}

tr_status tc_compress(const tr_model* m, const void* x, int64_t n, void* tokens, cudaStream_t st) {
  const int* c = m->desc.comp_dims;
  if ((uintptr_t)x % 16 || (uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "x/tokens not 16-byte aligned");
  auto encode = get_encode();
  if (!encode) return fail(TR_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  CompParams p;
  memset(&p, 0, sizeof p);
  cuuint64_t gdim[2] = {(cuuint64_t)c[0], (cuuint64_t)n};
  cuuint64_t gstride[1] = {(cuuint64_t)c[0] * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = encode(&p.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box, estride,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TR_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  const uint8_t* img = static_cast<const uint8_t*>(m->tc_comp);
  p.w1 = img;
  p.w2 = img + (size_t)c[0] * c[1] * 2;
  p.w3 = p.w2 + (size_t)c[1] * c[2] * 2;
  p.vec = m->tc_comp_vec;
  p.out = static_cast<float*>(tokens);
  p.status = ds->status;
  TR_TRY(stream_counters(st, &p.claim));
  TR_CUDA_TRY(cudaMemsetAsync(p.claim, 0, sizeof(int), st));
  p.n = n;
  p.n_tiles = (int)((n + kM - 1) / kM);
  p.c0 = c[0];
  p.c1 = c[1];
  p.c2 = c[2];
  p.c3 = c[3];
  int dev = 0, sms = 148;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  TR_TRY(ensure_smem_attr((const void*)compress_kernel, SMEM_BYTES));
  compress_kernel<<<std::min(p.n_tiles, sms), 320, SMEM_BYTES, st>>>(p);
  TR_LAUNCH_CHECK("compress_kernel");
  return TR_OK;
}

}  // namespace tr
