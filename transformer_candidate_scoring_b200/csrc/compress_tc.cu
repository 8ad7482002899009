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
//
// A second variant (compress_gather_kernel, tr_compress_target_bags) takes the candidates'
// field bags instead of x: eight more warps compute each 64-column slice of x on chip (the
// weighted averages of TransRetrieval §3.2) into a ring of their own, claim the tiles, and
// leave W1 and W2 / W3 to the copy thread; the MMA and epilogue roles are the same code.
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

// Shared-memory plan of the two variants.
//  - Plain (x from global memory): R1 holds two stages of [x slice (16 KB) | W1 slice (<= 64 KB)];
//    R2 two stages of 64-wide W2 / W3 slices (32 KB).  The hidden activations of layers 1 and 2
//    (fp16, <= 128 KB) are written over R1 once a tile's first GEMM is done; the LayerNorm
//    exchange buffer (R1 + 128 KB) and the per-column vectors of the running epilogue
//    (R1 + 132 KB, 8 KB) sit in the part of the second stage that is idle from the end of a
//    tile's first GEMM until the next tile's loads, which wait for its last GEMM.
//  - Gathering (x built on chip from the bags): R1 holds two W1 slices (64 KB each) and the
//    hidden activations; x has a ring of its own (three 16 KB stages), so the gather warps run
//    ahead of the tile in flight; W2 / W3 go in 32-wide slices (16 KB stages) to make room.
template <bool G> struct CLayout;
template <> struct CLayout<false> {
  static constexpr int THREADS = 320, EPI0 = 2;   // warps 2-9 run the epilogues
  static constexpr int STAGE1 = 80 * 1024, W1_OFF = 16384;
  static constexpr int XR = 0, XSTAGE = 0;
  static constexpr int R2 = 2 * STAGE1, STAGE2 = 32 * 1024, KW2 = 64;
  static constexpr int XBUF = 128 * 1024, VEC = 132 * 1024;
  static constexpr int BAR = R2 + 2 * STAGE2;
};
template <> struct CLayout<true> {
  // five warpgroups: copy and MMA threads (warps 0-3), epilogues (4-11), gather (12-19);
  // launched at 96 registers a thread, the control warpgroup gives registers to the others
  static constexpr int THREADS = 640, EPI0 = 4, GW0 = 12;
  static constexpr int LAUNCH_REGS = 96, CTL_REGS = 32, EPI_REGS = 104, GATHER_REGS = 120;
  static constexpr int STAGE1 = 64 * 1024, W1_OFF = 0;
  static constexpr int XR = 2 * STAGE1, XSTAGE = 16 * 1024, NX = 2;
  static constexpr int R2 = XR + NX * XSTAGE, STAGE2 = 16 * 1024, KW2 = 32;
  static constexpr int XBUF = R2 + 2 * STAGE2, VEC = XBUF + 4096;
  // the tile's bag headers: kM * F + 1 offsets (int64), then kM * F table ids (F <= 8)
  static constexpr int HDR = VEC + 8192, HDR_TAB = HDR + (kM * 8 + 2) * 8;
  static constexpr int BAR = HDR_TAB + kM * 8 * 4;
};
template <bool G> constexpr int smem_bytes() { return CLayout<G>::BAR + 256 + 1024 + 1024; }
static_assert(128 * CLayout<true>::CTL_REGS + 256 * (CLayout<true>::EPI_REGS + CLayout<true>::GATHER_REGS) <=
                  CLayout<true>::THREADS * CLayout<true>::LAUNCH_REGS &&
              CLayout<true>::THREADS * CLayout<true>::LAUNCH_REGS <= 65536,
              "register split of the gathering variant");
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory plan");
constexpr int kGatherWarps = 8;
constexpr int kMaxGatherFields = 8;   // the header table holds kM * 8 bags

// The bags of the gathering variant: candidate c's F field bags are c*F .. c*F + F - 1
// (the layout tr_aggregate reads), each over one of the bf16 tables.
struct GatherArgs {
  const uint16_t* tab[TR_MAX_TABLES];
  int rows[TR_MAX_TABLES];     // min(rows, INT32_MAX): every int32 key is below it past that
  const int32_t* bag_table;
  const int64_t* offsets;
  const int32_t* keys;
  const float* weights;
  int n_tables, F, D;
};

struct CompParams {
  CUtensorMap xmap;            // x [n][c0] bf16, box {64, 128}, 128-byte swizzle (plain variant)
  const uint8_t* w1;           // [c0/64] slices of W1^T [c1 x 64]
  const uint8_t* w2;           // [c1/64] slices of W2^T [c2 x 64]
  const uint8_t* w3;           // [c2/64] slices of W3^T [c3 x 64]
  const float* vec;            // b1 a1 g1 be1 (c1 each), b2 a2 g2 be2 (c2 each), b3 (c3)
  float* out;                  // [n][c3]
  int* status;
  int* claim;                  // next unclaimed tile (zero at launch)
  long long n;
  int n_tiles, c0, c1, c2, c3;
  GatherArgs g;                // gathering variant only
};

struct CBars {
  uint32_t full1[2], empty1[2], full2[2], empty2[2], r1_free, mma, epi, drain, qsync[4], vsync;
  uint32_t tile_full[2], tile_empty[2], tile_slot[2];   // the claimed-tile ring
  uint32_t xfull[3], xempty[3];                         // the x ring (gathering variant)
  uint32_t gsync;                                       // rendezvous of the gather warps
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

// Long waits of the gathering variant suspend instead of spinning (its gather warps need the
// issue slots); the plain variant keeps the spinning wait.
template <bool G>
__device__ __forceinline__ bool cwait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  return G ? mbar_wait_idle(bar, parity, abort_flag) : mbar_wait(bar, parity, abort_flag);
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

// Copy thread.  Plain variant: claims the tiles, publishes them to the other roles and
// loads each x slice with its W1 slice.  Gathering variant: reads the tiles from the ring
// (the gather warps claim them) and loads only weights.
template <bool G>
__device__ void comp_producer(const CompParams& p, uint32_t r1, uint32_t r2, const CBars& b, volatile int* abort_flag) {
  using L = CLayout<G>;
  int s1 = 0, s2 = 0;
  uint32_t ph1 = 0, ph2 = 0, free_phase = 0;
  const uint32_t w1_bytes = p.c1 * 128, w2_bytes = p.c2 * L::KW2 * 2, w3_bytes = p.c3 * L::KW2 * 2;
  bool ok = true;
  bool pend1[2] = {false, false}, pend2[2] = {false, false};
  uint32_t par1[2] = {0, 0}, par2[2] = {0, 0};
  int ts = 0;
  uint32_t tph = 0;
  for (int tile = G ? 0 : atomicAdd(p.claim, 1); ok;) {
    int cur;
    if constexpr (G) {
      cur = next_tile(b, ts, tph, abort_flag, ok);
    } else {
      // publish the tile (or the end) to the MMA and epilogue threads
      if (!(ok = mbar_wait(b.tile_empty[ts], tph ^ 1, abort_flag))) break;
      cur = tile < p.n_tiles ? tile : -1;
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(b.tile_slot[ts]), "r"(cur) : "memory");
      mbar_arrive(b.tile_full[ts]);
      if (++ts == 2) {
        ts = 0;
        tph ^= 1;
      }
    }
    if (cur < 0) break;
    // the stage buffers hold the previous tile's activations until its last GEMM is done
    if (!(ok = cwait<G>(b.r1_free, free_phase ^ 1, abort_flag))) break;
    free_phase ^= 1;
    for (int kc = 0; kc < p.c0 / 64 && ok; ++kc) {
      if (!(ok = cwait<G>(b.empty1[s1], ph1 ^ 1, abort_flag))) break;
      const uint32_t st = r1 + s1 * L::STAGE1;
      mbar_arrive_expect_tx(b.full1[s1], (G ? 0 : kM * 64 * 2) + w1_bytes);
      if constexpr (!G) tma_load_2d(st, &p.xmap, kc * 64, cur * kM, b.full1[s1]);
      bulk_g2s(st + L::W1_OFF, p.w1 + (size_t)kc * w1_bytes, w1_bytes, b.full1[s1]);
      pend1[s1] = true;
      par1[s1] = ph1;
      if (++s1 == 2) { s1 = 0; ph1 ^= 1; }
    }
    // W2 / W3 in KW2-wide slices: the images hold 64-wide slices one after the other, and
    // the first and second 32 columns of one are its two halves, so slice j of width KW2
    // starts j slices in
    for (int j = 0; j < p.c1 / L::KW2 + p.c2 / L::KW2 && ok; ++j) {
      if (!(ok = cwait<G>(b.empty2[s2], ph2 ^ 1, abort_flag))) break;
      const bool is2 = j < p.c1 / L::KW2;
      const uint32_t bytes = is2 ? w2_bytes : w3_bytes;
      const uint8_t* src = is2 ? p.w2 + (size_t)j * w2_bytes : p.w3 + (size_t)(j - p.c1 / L::KW2) * w3_bytes;
      mbar_arrive_expect_tx(b.full2[s2], bytes);
      bulk_g2s(r2 + s2 * L::STAGE2, src, bytes, b.full2[s2]);
      pend2[s2] = true;
      par2[s2] = ph2;
      if (++s2 == 2) { s2 = 0; ph2 ^= 1; }
    }
    if constexpr (!G) tile = atomicAdd(p.claim, 1);
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

template <bool G>
__device__ void comp_mma(const CompParams& p, uint32_t tmem, uint32_t r1, uint32_t r2, const CBars& b,
                         volatile int* abort_flag) {
  using L = CLayout<G>;
  constexpr int KS = L::KW2 / 16;   // MMAs per W2 / W3 slice
  int s1 = 0, s2 = 0, sx = 0;
  uint32_t ph1 = 0, ph2 = 0, phx = 0, epi_phase = 0;
  bool ok = true;
  const int n1 = std::min(p.c1, 256);
  // layer 1 multiplies bf16 x by bf16 W1; layers 2 and 3 fp16 activations by fp16 weights
  const uint32_t id1 = idesc_bf16(kM, n1), id2 = idesc_f16c(kM, p.c2), id3 = idesc_f16c(kM, p.c3);
  auto wait_epi = [&]() {
    ok = ok && cwait<G>(b.epi, epi_phase, abort_flag);
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
      if (!(ok = cwait<G>(b.full1[s1], ph1, abort_flag))) break;
      if constexpr (G) {
        if (!(ok = mbar_wait_idle(b.xfull[sx], phx, abort_flag))) break;
      }
      tc_fence_after();
      const uint32_t xa = G ? r1 + L::XR + sx * L::XSTAGE : r1 + s1 * L::STAGE1;
      const uint32_t wb = r1 + s1 * L::STAGE1 + L::W1_OFF;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        for (int nh = 0; nh < p.c1 / n1; ++nh)
          mma_bf16(tmem + nh * n1, sdesc_sw128(xa + kk * 32),
                   sdesc(wb + kk * 2 * p.c1 * 16 + nh * (n1 / 8) * 128, p.c1 * 16, 128), id1,
                   (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(b.empty1[s1]);
      if (++s1 == 2) { s1 = 0; ph1 ^= 1; }
      if constexpr (G) {
        mma_commit(b.xempty[sx]);
        if (++sx == L::NX) { sx = 0; phx ^= 1; }
      }
    }
    if (!ok) break;
    mma_commit(b.mma);
    if (!wait_epi()) break;                                // h1 (fp16) in R1
    for (int kc = 0; kc < p.c1 / L::KW2 && ok; ++kc) {
      if (!(ok = cwait<G>(b.full2[s2], ph2, abort_flag))) break;
      tc_fence_after();
      const uint32_t wb = r2 + s2 * L::STAGE2;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        mma_bf16(tmem, sdesc(r1 + (KS * kc + kk) * 2 * kM * 16, kM * 16, 128),
                 sdesc(wb + kk * 2 * p.c2 * 16, p.c2 * 16, 128), id2, (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(b.empty2[s2]);
      if (++s2 == 2) { s2 = 0; ph2 ^= 1; }
    }
    if (!ok) break;
    mma_commit(b.mma);
    if (!wait_epi()) break;                                // h2 (fp16) in R1
    for (int kc = 0; kc < p.c2 / L::KW2 && ok; ++kc) {
      if (!(ok = cwait<G>(b.full2[s2], ph2, abort_flag))) break;
      tc_fence_after();
      const uint32_t wb = r2 + s2 * L::STAGE2;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        mma_bf16(tmem + 256, sdesc(r1 + (KS * kc + kk) * 2 * kM * 16, kM * 16, 128),
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

template <bool G>
__device__ void comp_epilogue(const CompParams& p, uint32_t tmem, uint32_t r1, const CBars& b, float* svec,
                              float* sb3, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  CEpi e;
  e.q = warp & 3;
  e.m = e.q * 32 + lane;
  e.hf = (warp - CLayout<G>::EPI0) >> 2;
  e.trow = tmem + ((uint32_t)(e.q * 32) << 16);
  e.rowoff = (e.m >> 3) * 128 + (e.m & 7) * 16;
  e.xbuf = r1 + CLayout<G>::XBUF;
  e.qbar = b.qsync[e.q];
  e.ph_q = 0;
  e.abort_flag = abort_flag;
  e.ok = true;
  const float* v1 = p.vec;
  const float* v2 = p.vec + 4 * p.c1;
  const float* b3 = v2 + 4 * p.c2;
  const int et = threadIdx.x - 32 * CLayout<G>::EPI0;   // 0 .. 255
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
    e.ok = e.ok && cwait<G>(b.mma, mma_phase, abort_flag);
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

// a0 += w * x0, a1 += w * x1 as one packed fp32x2 FMA, each lane rounded as fmaf: the
// accumulation of tr_aggregate, so that the x rows built on chip equal its tokens bit for bit
__device__ __forceinline__ void fma2_acc(float& a0, float& a1, float w, float x0, float x1) {
  asm("{\n\t.reg .b64 a, x, w;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 x, {%3, %4};\n\tmov.b64 w, {%2, %2};\n\t"
      "fma.rn.f32x2 a, w, x, a;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(w), "f"(x0), "f"(x1));
}

__device__ __forceinline__ uint4 ld_row16(const uint16_t* q) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(q));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Gather warps of the gathering variant (TransRetrieval §3.2 feeding §3.3): the x row of a
// candidate is its F field tokens side by side, token f = sum_i v_i h(k_i) / sum_i v_i over
// the bag c*F + f.  Every 64-column slice of the tile in flight (field f, columns d0 .. d0+63
// of its token) is built in one stage of the x ring: eight lanes per bag, each owning 8
// columns (one 16-byte vector of every row), two bags per lane group at a time (a work item),
// so a group has up to 16 rows in flight.  Keys and weights are taken 8 at a time, one per
// lane, and broadcast by shuffle; rows are summed in bag order with fp32 FMAs and the weight
// sum is reduced across the 8 lanes, exactly as tr_aggregate does, then the token is rounded
// to bf16 and stored in the 128-byte-swizzled K-major layout the MMA reads.
// Latency: the tile's bag headers (offsets, table ids) are read into shared memory once per
// tile, and the next work item's first keys and weights are requested while the current
// item's rows are in flight, so an item costs about one row round trip.  Lane 0 of the first
// gather warp claims the tiles and publishes them to the other roles.
__device__ void comp_gather(const CompParams& p, uint32_t xr, uint8_t* hdr, const CBars& b, volatile int* abort_flag) {
  using L = CLayout<true>;
  const GatherArgs& g = p.g;
  constexpr int NGRP = 4 * kGatherWarps;   // lane groups
  constexpr int NPAIR = kM / NGRP / 2;     // work items of a group per slice
  const int lane = threadIdx.x & 31, gw = (threadIdx.x >> 5) - L::GW0;
  const int cl = lane & 7, grp = gw * 4 + (lane >> 3);
  const int gt = threadIdx.x - 32 * L::GW0;   // 0 .. 255
  const int F = g.F, per_field = g.D / 64, nkc = p.c0 / 64;
  const int nb = kM * F;                      // bags per tile
  const int64_t* s_off = reinterpret_cast<const int64_t*>(hdr);
  const int* s_tab = reinterpret_cast<const int*>(hdr + (L::HDR_TAB - L::HDR));
  const bool claimer = gw == 0 && lane == 0;
  bool ok = true, bad = false;
  int ts = 0, sx = 0;
  uint32_t tph = 0, phx = 0, gph = 0;
  // bounded rendezvous of the gather warps
  auto gsync = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(b.gsync);
    ok = ok && mbar_wait(b.gsync, gph, abort_flag);
    gph ^= 1;
    ok = __all_sync(0xffffffffu, ok);
    return ok;
  };
  for (;;) {
    if (claimer) {
      ok = ok && mbar_wait(b.tile_empty[ts], tph ^ 1, abort_flag);
      const int t = ok ? atomicAdd(p.claim, 1) : -1;
      const int pub = t >= 0 && t < p.n_tiles ? t : -1;
      asm volatile("st.shared.b32 [%0], %1;" ::"r"(b.tile_slot[ts]), "r"(pub) : "memory");
      mbar_arrive(b.tile_full[ts]);
    }
    const int tile = next_tile(b, ts, tph, abort_flag, ok);
    if (__any_sync(0xffffffffu, tile < 0)) break;
    // the tile's headers, once every gather warp is done with the previous tile's
    if (!gsync()) break;
    const long long bag0 = (long long)tile * nb;
    const int nb_here = (int)min((long long)nb, p.n * F - bag0);
    for (int i = gt; i <= nb_here; i += 32 * kGatherWarps)
      const_cast<int64_t*>(s_off)[i] = __ldg(g.offsets + bag0 + i);
    for (int i = gt; i < nb_here; i += 32 * kGatherWarps) const_cast<int*>(s_tab)[i] = __ldg(g.bag_table + bag0 + i);
    if (!gsync()) break;
    // header of bag slot j (0, 1) of work item (kc, pr): whether the candidate exists, its
    // table, first key and key count
    auto header = [&](int kc, int pr, int j, int& t, int64_t& s0, int& n) {
      const int r = grp + NGRP * (2 * pr + j);
      const int lb = r * F + kc / per_field;
      t = 0;
      s0 = 0;
      n = 0;
      if (lb >= nb_here) return false;
      t = s_tab[lb];
      s0 = s_off[lb];
      n = (int)(s_off[lb + 1] - s0);
      return true;
    };
    // first key chunk of work item (kc, pr), one key and weight per lane (k = -1: none)
    auto first_keys = [&](int kc, int pr, int (&k)[2], float (&v)[2]) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        int t, n;
        int64_t s0;
        const bool live = header(kc, pr, j, t, s0, n);
        k[j] = -1;
        v[j] = 0.f;
        if (live && t >= 0 && t < g.n_tables && cl < n) {
          k[j] = __ldg(g.keys + s0 + cl);
          v[j] = __ldg(g.weights + s0 + cl);
        }
      }
    };
    int kn[2];
    float vn[2];
    first_keys(0, 0, kn, vn);
    for (int kc = 0; kc < nkc; ++kc) {
      const int d0 = (kc % per_field) * 64;
      ok = ok && mbar_wait_idle(b.xempty[sx], phx ^ 1, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const uint32_t xs = xr + sx * L::XSTAGE;
#pragma unroll 1
      for (int pr = 0; pr < NPAIR; ++pr) {
        // a bag naming no table gets no rows: its weight sum stays 0 and its token 0
        int n[2], tb[2];
        const uint16_t* tp[2];
        int k[2] = {kn[0], kn[1]};
        float v[2] = {vn[0], vn[1]};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          int64_t s0;
          const bool live = header(kc, pr, j, tb[j], s0, n[j]);
          const bool badt = live && (tb[j] < 0 || tb[j] >= g.n_tables);
          bad |= badt;
          if (badt) n[j] = 0;
          if (n[j] == 0) tb[j] = 0;
          tp[j] = g.tab[tb[j]] + d0 + cl * 8;
        }
        const int n_max = __reduce_max_sync(0xffffffffu, max(n[0], n[1]));
        float acc[2][8], ws[2] = {0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
        for (int base = 0; base < n_max; base += 8) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int cnt = n[j] - base;
            if (base > 0) {   // chunks after the first (bags of more than 8 keys)
              k[j] = -1;
              v[j] = 0.f;
              if (cl < cnt) {
                int t;
                int64_t s0;
                int nn;
                header(kc, pr, j, t, s0, nn);
                k[j] = __ldg(g.keys + s0 + base + cl);
                v[j] = __ldg(g.weights + s0 + base + cl);
              }
            }
            if (cl >= cnt) {
              k[j] = -1;
              v[j] = 0.f;
            } else if (k[j] < 0 || k[j] >= g.rows[tb[j]]) {
              bad = true;
              k[j] = -1;
              v[j] = 0.f;
            }
            ws[j] += v[j];
          }
          const int cnt_max = min(n_max - base, 8);   // warp-uniform
          // a row past the bag's end or with a rejected key has k = -1 and weight 0
          uint4 raw[2][8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int kk = __shfl_sync(0xffffffffu, k[j], u, 8);
              raw[j][u] = u < cnt_max && kk >= 0 ? ld_row16(tp[j] + (int64_t)kk * g.D) : make_uint4(0, 0, 0, 0);
            }
          if (base == 0) {   // the next work item's first keys, while these rows are in flight
            const int nkc2 = pr + 1 < NPAIR ? kc : kc + 1, npr = pr + 1 < NPAIR ? pr + 1 : 0;
            if (nkc2 < nkc) first_keys(nkc2, npr, kn, vn);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (u >= cnt_max) break;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const float w = __shfl_sync(0xffffffffu, v[j], u, 8);
              const uint32_t q[4] = {raw[j][u].x, raw[j][u].y, raw[j][u].z, raw[j][u].w};
#pragma unroll
              for (int h = 0; h < 4; ++h)
                fma2_acc(acc[j][2 * h], acc[j][2 * h + 1], w, __uint_as_float(q[h] << 16),
                         __uint_as_float(q[h] & 0xFFFF0000u));
            }
          }
        }
        if (n_max == 0) {   // no rows anywhere in the warp: the next keys are still needed
          const int nkc2 = pr + 1 < NPAIR ? kc : kc + 1, npr = pr + 1 < NPAIR ? pr + 1 : 0;
          if (nkc2 < nkc) first_keys(nkc2, npr, kn, vn);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int off = 4; off > 0; off >>= 1) ws[j] += __shfl_xor_sync(0xffffffffu, ws[j], off);
          const float inv = ws[j] != 0.f ? 1.f / ws[j] : 0.f;
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = acc[j][e] * inv;
          const int r = grp + NGRP * (2 * pr + j);
          st_shared_v4(xs + (r >> 3) * 1024 + (r & 7) * 128 + ((cl ^ (r & 7)) << 4), pack_bf2(o[0], o[1]),
                       pack_bf2(o[2], o[3]), pack_bf2(o[4], o[5]), pack_bf2(o[6], o[7]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(b.xfull[sx]);
      if (++sx == L::NX) {
        sx = 0;
        phx ^= 1;
      }
    }
    if (!ok) break;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, STATUS_KEY_RANGE);
}

template <bool G>
__device__ __forceinline__ void compress_body(const CompParams& p) {
  using L = CLayout<G>;
  extern __shared__ uint8_t smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t r1 = base, r2 = base + L::R2, bar0 = base + L::BAR;
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
  for (int s = 0; s < 3; ++s) {
    b.xfull[s] = bar0 + 192 + 8 * s;
    b.xempty[s] = bar0 + 216 + 8 * s;
  }
  b.gsync = bar0 + 240;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::BAR + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::BAR + 136);
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
      // readers: the MMA thread and every epilogue thread; with gathering also the copy
      // thread and every gather thread
      mbar_init(b.tile_empty[s], G ? 2 + 256 + 32 * kGatherWarps : 1 + 256);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(b.xfull[s], kGatherWarps);
      mbar_init(b.xempty[s], 1);
    }
    mbar_init(b.gsync, kGatherWarps);
    *abort_flag = 0;
    mbar_fence_init();
    if constexpr (!G) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.xmap)) : "memory");
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
  float* svec = reinterpret_cast<float*>(gbase + L::VEC);
  float* sb3 = reinterpret_cast<float*>(gbase + L::BAR + 256);
  if constexpr (G) {
    // each role runs inside its own register budget
    if (warp < 4) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(CLayout<true>::CTL_REGS));
      if (warp == 0 && lane == 0) comp_producer<true>(p, r1, r2, b, abort_flag);
      if (warp == 1 && lane == 0) comp_mma<true>(p, tmem, r1, r2, b, abort_flag);
    } else if (warp < CLayout<true>::GW0) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(CLayout<true>::EPI_REGS));
      comp_epilogue<true>(p, tmem, r1, b, svec, sb3, abort_flag);
    } else {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(CLayout<true>::GATHER_REGS));
      comp_gather(p, r1 + L::XR, gbase + L::HDR, b, abort_flag);
    }
  } else {
    if (warp == 0) {
      if (lane == 0) comp_producer<false>(p, r1, r2, b, abort_flag);
    } else if (warp == 1) {
      if (lane == 0) comp_mma<false>(p, tmem, r1, r2, b, abort_flag);
    } else {
      comp_epilogue<false>(p, tmem, r1, b, svec, sb3, abort_flag);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, STATUS_KERNEL_TIMEOUT);
}

__global__ void __launch_bounds__(320, 1) compress_kernel(const __grid_constant__ CompParams p) {
  compress_body<false>(p);
}

__global__ void __launch_bounds__(640, 1) compress_gather_kernel(const __grid_constant__ CompParams p) {
  compress_body<true>(p);
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

namespace {

// Weight images, vectors, work counter and sizes of one launch (the x source aside).
tr_status comp_params(const tr_model* m, int64_t n, void* tokens, cudaStream_t st, CompParams& p, int& sms) {
  const int* c = m->desc.comp_dims;
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
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
  int dev = 0;
  sms = 148;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  return TR_OK;
}

template <bool G>
tr_status comp_launch(const CompParams& p, int sms, cudaStream_t st) {
  const void* k = G ? (const void*)compress_gather_kernel : (const void*)compress_kernel;
  TR_TRY(ensure_smem_attr(k, smem_bytes<G>()));
  if (G)
    compress_gather_kernel<<<std::min(p.n_tiles, sms), CLayout<G>::THREADS, smem_bytes<G>(), st>>>(p);
  else
    compress_kernel<<<std::min(p.n_tiles, sms), CLayout<G>::THREADS, smem_bytes<G>(), st>>>(p);
  TR_LAUNCH_CHECK(G ? "compress_gather_kernel" : "compress_kernel");
  return TR_OK;
}

}  // namespace

tr_status tc_compress(const tr_model* m, const void* x, int64_t n, void* tokens, cudaStream_t st) {
  const int* c = m->desc.comp_dims;
  if ((uintptr_t)x % 16 || (uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "x/tokens not 16-byte aligned");
  auto encode = get_encode();
  if (!encode) return fail(TR_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
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
  int sms = 148;
  TR_TRY(comp_params(m, n, tokens, st, p, sms));
  return comp_launch<false>(p, sms, st);
}

bool tc_comp_bags_supported(const tr_model* m) {
  const int D = m->desc.D;
  return tc_comp_supported(m) && D % 64 == 0 && m->desc.n_target_fields <= kMaxGatherFields &&
         m->desc.comp_dims[0] == m->desc.n_target_fields * D;
}

tr_status tc_compress_bags(const tr_model* m, const tr_table* tables, int n_tables, const int32_t* bag_table,
                           const int64_t* offsets, const int32_t* keys, const float* weights, int64_t n,
                           void* tokens, cudaStream_t st) {
  if ((uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "tokens not 16-byte aligned");
  CompParams p;
  memset(&p, 0, sizeof p);
  for (int i = 0; i < n_tables; ++i) {
    p.g.tab[i] = static_cast<const uint16_t*>(tables[i].data);
    p.g.rows[i] = (int)std::min<int64_t>(tables[i].n_rows, INT32_MAX);
  }
  p.g.bag_table = bag_table;
  p.g.offsets = offsets;
  p.g.keys = keys;
  p.g.weights = weights;
  p.g.n_tables = n_tables;
  p.g.F = m->desc.n_target_fields;
  p.g.D = m->desc.D;
  int sms = 148;
  TR_TRY(comp_params(m, n, tokens, st, p, sms));
  return comp_launch<true>(p, sms, st);
}

}  // namespace tr
