// Fused candidate stack on tcgen05 tensor cores (TransRetrieval §3.3, deployment section
// "Hardware-aware inference optimization").
//
// One persistent CTA per SM walks 128-candidate tiles; a tile never mixes requests, so
// every row of a tile attends to the same user K/V (the paper's "expand" broadcast: the
// request's cache is staged once per tile and layer, never replicated per candidate).
// The whole N-layer stack runs with the tile on chip:
//
//   TMEM (512 fp32 columns x 128 lanes, lane = candidate row)
//     [  0,128)  Y, the residual stream; the O and FFN2 GEMMs accumulate into it in place
//     [128,256)  Q accumulator -> per-head-group scores S -> FFN hidden (first half)
//     [256,384)  K accumulator -> attention output O       -> FFN hidden (second half)
//     [384,512)  the candidate's own V accumulator (kept until the attention epilogue)
//   shared memory (224 KB)
//     A      [128 x 128] bf16  LN1 output -> Q -> attention output -> LN2 output
//     P/H    [128 x 256] bf16  softmax numerators of one head group / ReLU(FFN hidden)
//     KV     the request's K and V^T images of the current layer (L_u <= 128)
//     ring   4 x 16 KB weight chunks ([128 out x 64 in] slices), streamed by the TMA engine
//
// Warp roles: warp 0 issues bulk copies (weights in consumption order, the K/V images
// once per tile and layer), warp 1 issues tcgen05.mma from one thread, warps 2-5 are the
// epilogue (one TMEM lane quadrant each; thread = candidate row, so LayerNorm and the
// per-head softmax need no cross-thread reduction).  LayerNorm gains/shifts and the
// softmax scale (1/sqrt(d_h), times log2 e for exp2) are folded into the weights when the
// model is built; the O and FFN2 biases are carried as a per-column offset of Y that the
// next LayerNorm adds back.  Every wait is bounded: a stalled barrier sets an error bit
// and the kernel unwinds, releasing its tensor memory.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "model.cuh"
#include "tc_common.cuh"

namespace tr {

tr_status simt_score(const tr_model* m, const void* tokens, int64_t c0, int64_t c1, const void* kv, int L_u,
                     int domain, float* scores, cudaStream_t st);

namespace {

using namespace tc;

constexpr int kD = 128, kH = 256, kM = 128;
constexpr int kChunk = 16384;                 // [128 x 64] bf16 weight slice
constexpr int kStages = 4;
constexpr int kChunksPerLayer = 16;
constexpr int kVecPerLayer = 9 * kD + kH;     // c1, g1, be1, bq*qs, bk, bv, c2, g2, be2, b1
constexpr float kQScale = 0.25f * 1.44269504088896341f;  // 1/sqrt(d_h) * log2(e)
constexpr int kVecFinal = 2 * kD + 16;        // cf, w, b
constexpr int kMaxLpTc = 128;

constexpr int OFF_A = 0;
constexpr int OFF_PH = OFF_A + kM * kD * 2;             // 32 KB
constexpr int OFF_KV = OFF_PH + kM * kH * 2;            // +64 KB
constexpr int OFF_RING = OFF_KV + 2 * kMaxLpTc * kD * 2;  // +64 KB
constexpr int OFF_BAR = OFF_RING + kStages * kChunk;    // +64 KB
constexpr int SMEM_BYTES = OFF_BAR + 128;


struct ReqInfo {
  const uint8_t* kv;
  long long cand_off;
  long long n;
  int tile_off;
  int L_u;
  int domain;
  int pad;
};

struct StackParams {
  const __nv_bfloat16* tokens;
  float* scores;
  const uint8_t* wimg;       // [n_layer][16][kChunk]
  const float* vec;          // [n_layer][kVecPerLayer] + [kVecFinal]
  const float* domain_emb;   // [n_domains][D]
  int* status;
  int n_layer;
  int n_tiles;
  int R;
  const float* utokens;      // user-side mode: fp32 user tokens [L_u][D]
  uint8_t* kv_out;           // user-side mode: the request's K/V cache
  ReqInfo req[TR_MAX_REQUESTS];
};

struct TileInfo {
  int r, rows, L_u, Lp, hg, ng;
  long long row0;
};

__device__ __forceinline__ TileInfo tile_info(const StackParams& p, int tile) {
  int r = 0;
  while (r + 1 < p.R && tile >= p.req[r + 1].tile_off) ++r;
  TileInfo t;
  t.r = r;
  t.row0 = p.req[r].cand_off + (long long)(tile - p.req[r].tile_off) * kM;
  t.rows = (int)min((long long)kM, p.req[r].cand_off + p.req[r].n - t.row0);
  t.L_u = p.req[r].L_u;
  t.Lp = (t.L_u + 15) & ~15;
  // heads per score group: the group's scores fill at most 128 TMEM columns
  t.hg = t.Lp <= 16 ? 8 : t.Lp <= 32 ? 4 : t.Lp <= 64 ? 2 : 1;
  t.ng = t.Lp == 0 ? 0 : 8 / t.hg;
  return t;
}

struct Bars {
  uint32_t full[kStages], empty[kStages], kv_full, kv_empty, mma, epi, drain, esync;
};

// ------------------------------------------------------------------ producer (warp 0, one thread)
template <bool PF>
__device__ void producer(const StackParams& p, uint32_t ring, uint32_t kvbuf, const Bars& b, volatile int* abort_flag) {
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0;
  bool pending[kStages] = {false, false, false, false};
  uint32_t pend_parity[kStages] = {0, 0, 0, 0};
  bool kv_pending = false;
  uint32_t kv_pend_parity = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    for (int l = 0; l < p.n_layer && ok; ++l) {
      const uint8_t* wl = p.wimg + (size_t)l * kChunksPerLayer * kChunk;
      for (int c = 0; c < kChunksPerLayer && ok; ++c) {
        if (!PF && c == 6) {  // the request's K/V images go in between the QKV and O weights
          if (!(ok = mbar_wait(b.kv_empty, kv_phase ^ 1, abort_flag))) break;
          const uint32_t bytes = 2u * t.Lp * kD * 2u;
          if (bytes) {
            mbar_arrive_expect_tx(b.kv_full, bytes);
            bulk_g2s(kvbuf, p.req[t.r].kv + (size_t)l * bytes, bytes, b.kv_full);
            kv_pending = true;
            kv_pend_parity = kv_phase;
          } else {
            mbar_arrive(b.kv_full);
          }
          kv_phase ^= 1;
        }
        if (!(ok = mbar_wait(b.empty[stage], phase ^ 1, abort_flag))) break;
        mbar_arrive_expect_tx(b.full[stage], kChunk);
        bulk_g2s(ring + stage * kChunk, wl + (size_t)c * kChunk, kChunk, b.full[stage]);
        pending[stage] = true;
        pend_parity[stage] = phase;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }
  if (!ok) {  // unwinding: let the copies already issued land before the CTA exits
    for (int s = 0; s < kStages; ++s)
      if (pending[s])
        for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.full[s], pend_parity[s]) && globaltimer_ns() - t0 < 200000000ull;) {
        }
    if (kv_pending)
      for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.kv_full, kv_pend_parity) && globaltimer_ns() - t0 < 200000000ull;) {
      }
  }
}

// ------------------------------------------------------------------ MMA issuer (warp 1, one thread)
template <bool PF>
__device__ void mma_issuer(const StackParams& p, uint32_t tmem, uint32_t sA, uint32_t sPH, uint32_t sKV, uint32_t ring,
                           const Bars& b, volatile int* abort_flag) {
  constexpr uint32_t ID128 = idesc_bf16(kM, 128);
  constexpr uint32_t ID16 = idesc_bf16(kM, 16);
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0, epi_phase = 0;
  bool ok = true;
  auto wait_epi = [&]() {
    ok = ok && mbar_wait(b.epi, epi_phase, abort_flag);
    epi_phase ^= 1;
    tc_fence_after();
    return ok;
  };
  // one [128 x 64] weight chunk against A K-steps [ks0, ks0 + 4)
  auto chunk = [&](uint32_t a_base, int ks0, uint32_t dcol, bool acc_first) {
    if (!ok) return;
    if (!(ok = mbar_wait(b.full[stage], phase, abort_flag))) return;
    tc_fence_after();
    const uint32_t w = ring + stage * kChunk;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tmem + dcol, sdesc(a_base + (ks0 + kk) * 4096, 2048, 128), sdesc(w + kk * 4096, 2048, 128), ID128,
               (kk > 0 || acc_first) ? 1u : 0u);
    mma_commit(b.empty[stage]);
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  };
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    const uint32_t idS = idesc_bf16(kM, t.Lp > 0 ? t.Lp : 16);
    for (int l = 0; l < p.n_layer && ok; ++l) {
      if (!wait_epi()) break;                         // A = LN1(y)
      chunk(sA, 0, 128, false);                       // Q
      chunk(sA, 4, 128, true);
      chunk(sA, 0, 256, false);                       // K (own)
      chunk(sA, 4, 256, true);
      chunk(sA, 0, 384, false);                       // V (own)
      chunk(sA, 4, 384, true);
      mma_commit(b.mma);
      if (!wait_epi()) break;                         // A = Q (scaled, biased)
      if (!PF) {
        ok = ok && mbar_wait(b.kv_full, kv_phase, abort_flag);
        kv_phase ^= 1;
        tc_fence_after();
      }
      for (int g = 0; g < t.ng && ok; ++g) {
        for (int s = 0; s < t.hg; ++s) {
          const int h = g * t.hg + s;
          mma_bf16(tmem + 128 + s * t.Lp, sdesc(sA + h * 4096, 2048, 128),
                   sdesc(sKV + 2 * h * (t.Lp / 8) * 128, (t.Lp / 8) * 128, 128), idS, 0u);
        }
        mma_commit(b.mma);
        if (!wait_epi()) break;                       // P of this head group in P/H
        for (int s = 0; s < t.hg; ++s) {
          const int h = g * t.hg + s;
          const uint32_t pb = sPH + s * t.Lp * 256;
          const uint32_t vb = sKV + t.Lp * 256;
          for (int kk = 0; kk < t.Lp / 16; ++kk)
            mma_bf16(tmem + 256 + 16 * h, sdesc(pb + kk * 4096, 2048, 128),
                     sdesc(vb + (32 * kk + 2 * h) * 128, 2048, 128), ID16, kk > 0 ? 1u : 0u);
        }
      }
      if (!ok) break;
      if (!PF) mma_commit(b.kv_empty);
      mma_commit(b.mma);
      if (!wait_epi()) break;                         // A = attention output
      chunk(sA, 0, 0, true);                          // Y += attn Wo
      chunk(sA, 4, 0, true);
      mma_commit(b.mma);
      if (!wait_epi()) break;                         // A = LN2(y)
      chunk(sA, 0, 128, false);                       // hidden[:, 0:128]
      chunk(sA, 4, 128, true);
      chunk(sA, 0, 256, false);                       // hidden[:, 128:256]
      chunk(sA, 4, 256, true);
      mma_commit(b.mma);
      if (!wait_epi()) break;                         // P/H = ReLU(hidden)
      for (int q = 0; q < 4; ++q) chunk(sPH, 4 * q, 0, true);  // Y += H W2
      mma_commit(b.mma);
    }
  }
  // drain every MMA still in flight before the tensor memory is released
  mma_commit(b.drain);
  for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.drain, 0) && globaltimer_ns() - t0 < 500000000ull;) {
  }
}

// ------------------------------------------------------------------ epilogue (warps 2-5)
__device__ __forceinline__ void ln_rows_to_smem(float* y, uint32_t sA, int m, const float* g, const float* be) {
  float mean = 0.f;
#pragma unroll
  for (int i = 0; i < kD; ++i) mean += y[i];
  mean *= (1.f / kD);
  float var = 0.f;
#pragma unroll
  for (int i = 0; i < kD; ++i) {
    const float d = y[i] - mean;
    var = fmaf(d, d, var);
  }
  const float rstd = rsqrtf(var * (1.f / kD) + kLnEps);
  const uint32_t rowoff = (m >> 3) * 128 + (m & 7) * 16;
#pragma unroll
  for (int kc = 0; kc < kD / 8; ++kc) {
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf((y[kc * 8 + i] - mean) * rstd, __ldg(g + kc * 8 + i), __ldg(be + kc * 8 + i));
    st_row8(sA + kc * 2048 + rowoff, v);
  }
}

__device__ __forceinline__ void load_y(uint32_t trow, float* y) {
#pragma unroll
  for (int c = 0; c < 8; ++c) tmem_ld16(trow + c * 16, y + c * 16);
  tmem_wait_ld();
  reg_fence<kD>(y);
}

// PF (user-side mode): the tile is the request's user tokens; each layer's K and V are
// the tile's own, written to the K/V images in shared memory and stored to the cache.
template <bool PF>
__device__ void epilogue(const StackParams& p, uint32_t tmem, uint32_t sA, uint32_t sPH, uint32_t sKV, const Bars& b,
                         volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3;
  const int m = q * 32 + lane;
  const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
  const uint32_t rowoff = (m >> 3) * 128 + (m & 7) * 16;
  uint32_t mma_phase = 0;
  bool ok = true;
  auto wait_mma = [&]() {
    ok = ok && mbar_wait(b.mma, mma_phase, abort_flag);
    mma_phase ^= 1;
    tc_fence_after();
    return ok;
  };
  auto signal = [&]() {
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(b.epi);
  };
  // rendezvous of the 128 epilogue threads (bounded, like every other wait)
  uint32_t esync_phase = 0;
  auto epi_sync = [&]() {
    mbar_arrive(b.esync);
    ok = ok && mbar_wait(b.esync, esync_phase, abort_flag);
    esync_phase ^= 1;
    return ok;
  };
  const float* vfin = p.vec + (size_t)p.n_layer * kVecPerLayer;
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    const float* sd = p.domain_emb + (size_t)p.req[t.r].domain * kD;
    // Y = t + s_d; rows past the request's end are zero and never stored
    if (PF) {
      const float* src = p.utokens + (t.row0 + m) * kD;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float yv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) yv[i] = (m < t.rows) ? __ldg(src + c * 16 + i) + __ldg(sd + c * 16 + i) : 0.f;
        tmem_st16(trow + c * 16, yv);
      }
      tmem_wait_st();
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(p.tokens + (t.row0 + m) * kD);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float yv[16];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 u = (m < t.rows) ? __ldg(src + 2 * c + hh) : make_uint4(0, 0, 0, 0);
          const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = c * 16 + hh * 8 + 2 * i;
            yv[hh * 8 + 2 * i] = (m < t.rows) ? __uint_as_float(w[i] << 16) + __ldg(sd + col) : 0.f;
            yv[hh * 8 + 2 * i + 1] = (m < t.rows) ? __uint_as_float(w[i] & 0xFFFF0000u) + __ldg(sd + col + 1) : 0.f;
          }
        }
        tmem_st16(trow + c * 16, yv);
      }
      tmem_wait_st();
    }

    for (int l = 0; l < p.n_layer && ok; ++l) {
      const float* vl = p.vec + (size_t)l * kVecPerLayer;
      const float *c1 = vl, *g1 = vl + kD, *be1 = vl + 2 * kD, *bq = vl + 3 * kD, *bk = vl + 4 * kD, *bv = vl + 5 * kD;
      const float *c2 = vl + 6 * kD, *g2 = vl + 7 * kD, *be2 = vl + 8 * kD, *b1 = vl + 9 * kD;
      // ---- LN1
      if (l > 0 && !wait_mma()) break;            // FFN2 of the previous layer done
      {
        float y[kD];
        load_y(trow, y);
#pragma unroll
        for (int i = 0; i < kD; ++i) y[i] += __ldg(c1 + i);
        ln_rows_to_smem(y, sA, m, g1, be1);
      }
      signal();
      // ---- Q, own K: the candidate's own score per head; Q to A
      if (!wait_mma()) break;
      float sself[8];
      if (PF && threadIdx.x == 64 && l > 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      if (PF && !epi_sync()) break;               // the K/V images are free to overwrite
      for (int h = 0; h < 8; ++h) {
        float qv[16], kv[16];
        tmem_ld16(trow + 128 + 16 * h, qv);
        tmem_ld16(trow + 256 + 16 * h, kv);
        tmem_wait_ld();
        reg_fence<16>(qv);
        reg_fence<16>(kv);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          qv[i] = fmaf(qv[i], kQScale, __ldg(bq + 16 * h + i));
          kv[i] += __ldg(bk + 16 * h + i);
          s = fmaf(qv[i], kv[i], s);
        }
        sself[h] = PF ? -INFINITY : s;
        st_row8(sA + (2 * h) * 2048 + rowoff, qv);
        st_row8(sA + (2 * h + 1) * 2048 + rowoff, qv + 8);
        if (PF) {
          // K image row m, V^T image column m (zero past L_u); the TMEM load is
          // warp-wide, only the stores depend on the row
          float vv[16];
          tmem_ld16(trow + 384 + 16 * h, vv);
          tmem_wait_ld();
          reg_fence<16>(vv);
          if (m < t.Lp) {
            const bool live = m < t.L_u;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              kv[i] = live ? kv[i] : 0.f;
              vv[i] = live ? vv[i] + __ldg(bv + 16 * h + i) : 0.f;
            }
            const uint32_t kb = sKV + (m >> 3) * 128 + (m & 7) * 16;
            st_row8(kb + (2 * h) * (t.Lp / 8) * 128, kv);
            st_row8(kb + (2 * h + 1) * (t.Lp / 8) * 128, kv + 8);
            const uint32_t vb = sKV + t.Lp * 256 + (m >> 3) * 2048 + (m & 7) * 2;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int d = 16 * h + i;
              const __nv_bfloat16 hv = __float2bfloat16_rn(vv[i]);
              asm volatile("st.shared.b16 [%0], %1;" ::"r"(vb + (d >> 3) * 128 + (d & 7) * 16),
                           "h"(*reinterpret_cast<const unsigned short*>(&hv))
                           : "memory");
            }
          }
        }
      }
      if (PF) {  // store this layer's K/V images to the cache with one bulk copy
        fence_proxy_async_smem();
        if (!epi_sync()) break;
        if (threadIdx.x == 64) {
          const uint32_t bytes = 2u * t.Lp * kD * 2u;
          asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                           p.kv_out + (size_t)l * bytes),
                       "r"(sKV), "r"(bytes)
                       : "memory");
          asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
      }
      signal();
      // ---- softmax over [user keys of the request, own key], one head group at a time
      float pself[8], linv[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        pself[h] = 1.f;
        linv[h] = 1.f;
      }
      for (int g = 0; g < t.ng && ok; ++g) {
        if (!wait_mma()) break;
        for (int s = 0; s < t.hg; ++s) {
          const int h = g * t.hg + s;
          // two passes over the head's scores in TMEM: the row max, then exp2 / sum / P
          const uint32_t scol = trow + 128 + s * t.Lp;
          float mx = sself[h];
          for (int c = 0; c < t.Lp / 16; ++c) {
            float sv[16];
            tmem_ld16(scol + c * 16, sv);
            tmem_wait_ld();
            reg_fence<16>(sv);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c * 16 + i < t.L_u) mx = fmaxf(mx, sv[i]);
          }
          float sum = 0.f;
          const uint32_t pb = sPH + s * t.Lp * 256 + rowoff;
          for (int c = 0; c < t.Lp / 16; ++c) {
            float sv[16];
            tmem_ld16(scol + c * 16, sv);
            tmem_wait_ld();
            reg_fence<16>(sv);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float e = (c * 16 + i < t.L_u) ? ex2(sv[i] - mx) : 0.f;
              sv[i] = e;
              sum += e;
            }
            st_row8(pb + (2 * c) * 2048, sv);
            st_row8(pb + (2 * c + 1) * 2048, sv + 8);
          }
          pself[h] = ex2(sself[h] - mx);
          linv[h] = 1.f / (sum + pself[h]);
        }
        signal();
      }
      if (!ok) break;
      // ---- attention output = (sum_j p_j v_j + p_self v_self) / l, to A
      if (!wait_mma()) break;
      for (int h = 0; h < 8; ++h) {
        float o[16], v[16];
        tmem_ld16(trow + 256 + 16 * h, o);
        tmem_ld16(trow + 384 + 16 * h, v);
        tmem_wait_ld();
        reg_fence<16>(o);
        reg_fence<16>(v);
        const float ps = pself[h], li = linv[h];
        const bool has_users = t.ng > 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float vs = v[i] + __ldg(bv + 16 * h + i);
          o[i] = ((has_users ? o[i] : 0.f) + ps * vs) * li;
        }
        st_row8(sA + (2 * h) * 2048 + rowoff, o);
        st_row8(sA + (2 * h + 1) * 2048 + rowoff, o + 8);
      }
      signal();
      // ---- LN2
      if (!wait_mma()) break;                     // Y += attn Wo done
      {
        float y[kD];
        load_y(trow, y);
#pragma unroll
        for (int i = 0; i < kD; ++i) y[i] += __ldg(c2 + i);
        ln_rows_to_smem(y, sA, m, g2, be2);
      }
      signal();
      // ---- ReLU(hidden + b1) to P/H
      if (!wait_mma()) break;
      for (int c = 0; c < kH / 16; ++c) {
        float hv[16];
        tmem_ld16(trow + 128 + 16 * c, hv);
        tmem_wait_ld();
        reg_fence<16>(hv);
#pragma unroll
        for (int i = 0; i < 16; ++i) hv[i] = fmaxf(hv[i] + __ldg(b1 + 16 * c + i), 0.f);
        st_row8(sPH + (2 * c) * 2048 + rowoff, hv);
        st_row8(sPH + (2 * c + 1) * 2048 + rowoff, hv + 8);
      }
      signal();
    }
    if (!ok) break;
    // ---- head: w . LN_f(y) + b
    if (!wait_mma()) break;
    if (PF) continue;
    float y[kD];
    load_y(trow, y);
    float mean = 0.f;
#pragma unroll
    for (int i = 0; i < kD; ++i) {
      y[i] += __ldg(vfin + i);
      mean += y[i];
    }
    mean *= (1.f / kD);
    float var = 0.f;
#pragma unroll
    for (int i = 0; i < kD; ++i) var = fmaf(y[i] - mean, y[i] - mean, var);
    const float rstd = rsqrtf(var * (1.f / kD) + kLnEps);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kD; ++i) acc = fmaf((y[i] - mean) * rstd, __ldg(vfin + kD + i), acc);
    if (m < t.rows) p.scores[t.row0 + m] = acc + __ldg(vfin + 2 * kD);
  }
}

template <bool PF>
__global__ void __launch_bounds__(192, 1) stack_kernel(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t sA = base + OFF_A, sPH = base + OFF_PH, sKV = base + OFF_KV, ring = base + OFF_RING;
  const uint32_t bar0 = base + OFF_BAR;
  Bars b;
  for (int s = 0; s < kStages; ++s) {
    b.full[s] = bar0 + 8 * s;
    b.empty[s] = bar0 + 8 * (kStages + s);
  }
  b.kv_full = bar0 + 8 * (2 * kStages);
  b.kv_empty = b.kv_full + 8;
  b.mma = b.kv_full + 16;
  b.epi = b.kv_full + 24;
  b.drain = b.kv_full + 32;
  b.esync = b.kv_full + 40;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 112);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 120);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b.full[s], 1);
      mbar_init(b.empty[s], 1);
    }
    mbar_init(b.kv_full, 1);
    mbar_init(b.kv_empty, 1);
    mbar_init(b.mma, 1);
    mbar_init(b.epi, 128);
    mbar_init(b.drain, 1);
    mbar_init(b.esync, 128);
    *abort_flag = 0;
    mbar_fence_init();
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
    if (lane == 0) producer<PF>(p, ring, sKV, b, abort_flag);
  } else if (warp == 1) {
    if (lane == 0) mma_issuer<PF>(p, tmem, sA, sPH, sKV, ring, b, abort_flag);
  } else {
    epilogue<PF>(p, tmem, sA, sPH, sKV, b, abort_flag);
    if (PF && threadIdx.x == 64) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, STATUS_KERNEL_TIMEOUT);
}

// ------------------------------------------------------------------ host: weight folding and images

// W^T slice [n0, n0+128) x [k0, k0+64) of W [K][N] (row-major, W[k][n]) in core-matrix layout.
void put_chunk(uint16_t* dst, const std::vector<double>& W, int N, int n0, int k0) {
  for (int n = 0; n < 128; ++n)
    for (int k = 0; k < 64; ++k) {
      const double v = W[(size_t)(k0 + k) * N + (n0 + n)];
      const size_t off = ((size_t)(k / 8) * 16 + n / 8) * 64 + (n % 8) * 8 + (k % 8);
      const float f = (float)v;
      uint32_t u;
      memcpy(&u, &f, 4);
      u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;  // round to nearest even
      dst[off] = (uint16_t)u;
    }
}

}  // namespace

bool tc_stack_supported(const tr_model* m) {
  const tr_model_desc& d = m->desc;
  return d.dtype == TR_BF16 && d.D == kD && d.ffn_hidden == kH && d.n_head == 8 && m->tc_stack;
}

tr_status tc_build_comp(tr_model* m, const tr_model_weights* w);

tr_status tc_build(tr_model* m, const tr_model_weights* w) {
  const tr_model_desc& d = m->desc;
  TR_TRY(tc_build_comp(m, w));
  if (!(d.dtype == TR_BF16 && d.D == kD && d.ffn_hidden == kH && d.n_head == 8)) return TR_OK;
  const int N = d.n_layer, D = kD, H = kH;
  std::vector<uint16_t> img((size_t)N * kChunksPerLayer * kChunk / 2);
  std::vector<float> vec((size_t)N * kVecPerLayer + kVecFinal, 0.f);
  std::vector<double> c(D, 0.0);
  auto dvec = [](const float* p, size_t n) { return std::vector<double>(p, p + n); };
  for (int l = 0; l < N; ++l) {
    // the weights go in unchanged (exact bf16 values); LayerNorm gains/shifts, biases and
    // the softmax scale stay fp32 and are applied by the epilogue
    const tr_layer_weights& L = w->layers[l];
    const auto Wq = dvec(L.Wq, D * D), Wk = dvec(L.Wk, D * D), Wv = dvec(L.Wv, D * D), Wo = dvec(L.Wo, D * D);
    const auto W1 = dvec(L.W1, D * H), W2 = dvec(L.W2, H * D);
    uint16_t* li = img.data() + (size_t)l * kChunksPerLayer * kChunk / 2;
    const size_t ce = kChunk / 2;
    put_chunk(li + 0 * ce, Wq, D, 0, 0);
    put_chunk(li + 1 * ce, Wq, D, 0, 64);
    put_chunk(li + 2 * ce, Wk, D, 0, 0);
    put_chunk(li + 3 * ce, Wk, D, 0, 64);
    put_chunk(li + 4 * ce, Wv, D, 0, 0);
    put_chunk(li + 5 * ce, Wv, D, 0, 64);
    put_chunk(li + 6 * ce, Wo, D, 0, 0);
    put_chunk(li + 7 * ce, Wo, D, 0, 64);
    put_chunk(li + 8 * ce, W1, H, 0, 0);
    put_chunk(li + 9 * ce, W1, H, 0, 64);
    put_chunk(li + 10 * ce, W1, H, 128, 0);
    put_chunk(li + 11 * ce, W1, H, 128, 64);
    for (int q = 0; q < 4; ++q) put_chunk(li + (12 + q) * ce, W2, D, 0, 64 * q);
    float* v = vec.data() + (size_t)l * kVecPerLayer;
    for (int j = 0; j < D; ++j) {
      v[j] = (float)c[j];                       // c1: biases accumulated in Y so far
      v[D + j] = L.ln1_g[j];
      v[2 * D + j] = L.ln1_b[j];
      v[3 * D + j] = (float)((double)L.bq[j] * (0.25 * 1.4426950408889634));
      v[4 * D + j] = L.bk[j];
      v[5 * D + j] = L.bv[j];
      c[j] += L.bo[j];
      v[6 * D + j] = (float)c[j];               // c2
      v[7 * D + j] = L.ln2_g[j];
      v[8 * D + j] = L.ln2_b[j];
      c[j] += L.b2[j];
    }
    for (int j = 0; j < H; ++j) v[9 * D + j] = L.b1[j];
  }
  float* vf = vec.data() + (size_t)N * kVecPerLayer;
  double bh = w->b_head;
  for (int j = 0; j < D; ++j) {
    vf[j] = (float)c[j];
    vf[D + j] = (float)((double)w->w_head[j] * w->lnf_g[j]);
    bh += (double)w->w_head[j] * w->lnf_b[j];
  }
  vf[2 * D] = (float)bh;
  const size_t img_bytes = img.size() * 2, vec_bytes = vec.size() * 4;
  const size_t total = img_bytes + ((vec_bytes + 255) & ~size_t(255));
  if (cudaMalloc(&m->tc_blob, total) != cudaSuccess) {
    cudaGetLastError();
    return fail(TR_ERR_NOMEM, "tensor-core weight images: allocation of %zu bytes failed", total);
  }
  m->tc_bytes = total;
  TR_CUDA_TRY(cudaMemcpy(m->tc_blob, img.data(), img_bytes, cudaMemcpyHostToDevice));
  TR_CUDA_TRY(cudaMemcpy((uint8_t*)m->tc_blob + img_bytes, vec.data(), vec_bytes, cudaMemcpyHostToDevice));
  m->tc_stack = m->tc_blob;
  m->tc_stack_layer_bytes = (size_t)kChunksPerLayer * kChunk;
  m->tc_vec = reinterpret_cast<const float*>((uint8_t*)m->tc_blob + img_bytes);
  m->tc_vec_layer_floats = kVecPerLayer;
  return TR_OK;
}

tr_status set_smem_attr(int dev) {
  static bool done[64] = {};
  if (dev < 0 || dev >= 64) return fail(TR_ERR_UNSUPPORTED, "device %d", dev);
  if (!done[dev]) {
    TR_CUDA_TRY(cudaFuncSetAttribute(stack_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    TR_CUDA_TRY(cudaFuncSetAttribute(stack_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    done[dev] = true;
  }
  return TR_OK;
}

tr_status tc_score(const tr_model* m, const void* tokens, int64_t n, const int64_t* req_offsets,
                   const void* const* kv, const int32_t* L_u, const int32_t* domain, int R, float* scores,
                   cudaStream_t st) {
  bool fits = true;
  for (int r = 0; r < R; ++r) fits = fits && L_u[r] <= kMaxLpTc;
  if (!fits) {  // long user sequences: CUDA-core path
    for (int r = 0; r < R; ++r)
      TR_TRY(simt_score(m, tokens, req_offsets[r], req_offsets[r + 1], kv[r], L_u[r], domain[r], scores, st));
    return TR_OK;
  }
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  StackParams p{};
  p.tokens = static_cast<const __nv_bfloat16*>(tokens);
  p.scores = scores;
  p.wimg = static_cast<const uint8_t*>(m->tc_stack);
  p.vec = m->tc_vec;
  p.domain_emb = m->domain_emb;
  p.status = ds->status;
  p.n_layer = m->desc.n_layer;
  p.R = R;
  int tiles = 0;
  for (int r = 0; r < R; ++r) {
    const int64_t nr = req_offsets[r + 1] - req_offsets[r];
    p.req[r].kv = static_cast<const uint8_t*>(kv[r]);
    p.req[r].cand_off = req_offsets[r];
    p.req[r].n = nr;
    p.req[r].tile_off = tiles;
    p.req[r].L_u = L_u[r];
    p.req[r].domain = domain[r];
    if ((uintptr_t)kv[r] % 16 && L_u[r] > 0 && nr > 0) return fail(TR_ERR_INVALID_ARG, "kv[%d] is not 16-byte aligned", r);
    tiles += (int)((nr + kM - 1) / kM);
  }
  if ((uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "tokens not 16-byte aligned");
  p.n_tiles = tiles;
  if (tiles == 0) return TR_OK;
  int dev = 0, sms = 148;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  TR_TRY(set_smem_attr(dev));
  const int grid = std::min(tiles, sms);
  stack_kernel<false><<<grid, 192, SMEM_BYTES, st>>>(p);
  TR_LAUNCH_CHECK("stack_kernel");
  return TR_OK;
}

bool tc_prefill_supported(const tr_model* m, int L_u) { return tc_stack_supported(m) && L_u <= kMaxLpTc; }

// User side of one request through the same kernel (one CTA, the user tokens as its tile).
tr_status tc_prefill(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv, cudaStream_t st) {
  if ((uintptr_t)kv % 16 || (uintptr_t)user_tokens % 16)
    return fail(TR_ERR_INVALID_ARG, "user_tokens / kv not 16-byte aligned");
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  StackParams p{};
  p.wimg = static_cast<const uint8_t*>(m->tc_stack);
  p.vec = m->tc_vec;
  p.domain_emb = m->domain_emb;
  p.status = ds->status;
  p.n_layer = m->desc.n_layer;
  p.R = 1;
  p.n_tiles = 1;
  p.utokens = user_tokens;
  p.kv_out = static_cast<uint8_t*>(kv);
  p.req[0].cand_off = 0;
  p.req[0].n = L_u;
  p.req[0].tile_off = 0;
  p.req[0].L_u = L_u;
  p.req[0].domain = domain;
  int dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_TRY(set_smem_attr(dev));
  stack_kernel<true><<<1, 192, SMEM_BYTES, st>>>(p);
  TR_LAUNCH_CHECK("stack_kernel (user side)");
  return TR_OK;
}


}  // namespace tr
