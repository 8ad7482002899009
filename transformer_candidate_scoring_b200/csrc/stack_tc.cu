// Fused candidate stack on tcgen05 tensor cores (TransRetrieval §3.3, deployment section
// "Hardware-aware inference optimization").
//
// One persistent CTA per SM walks 128-candidate tiles; a tile never mixes requests, so
// every row of a tile attends to the same user K/V (the paper's "expand" broadcast: the
// request's cache is staged once per tile and layer, never replicated per candidate).
// The whole N-layer stack runs with the tile on chip:
//
//   TMEM (512 fp32 columns x 128 lanes, lane = candidate row)
//     [  0,128)  Y, the residual stream; the O and FFN2 GEMMs (and their biases)
//                accumulate into it in place
//     [128,256)  Q accumulator -> score buffer 0 (softmax numerators written over the scores
//                as bf16, the A operand of P V) -> FFN hidden [0,128)
//     [256,384)  K accumulator -> score buffer 1 (same) -> FFN hidden [128,256)
//     [384,512)  V accumulator -> attention output O (the candidate's own V moves to
//                registers as bf16 first) -> ReLU(hidden) as bf16, the A operand of W2
//   shared memory
//     A      [128 x 128] bf16  LN1 output -> Q -> attention output -> LN2 output
//     KV     the request's K and V^T images of the current layer (up to 64 KB)
//     ring   3 x 36 KB: a [128 out x 128 in] weight block plus its [128 x 16] bias tile;
//            streamed by the TMA engine in consumption order
//     ones   the [128 x 16] A operand that turns a bias tile into "+ bias" in one MMA
//     vec    LayerNorm gains/shifts of every layer and the folded head weight (<= 5 layers)
//
// Attention runs per head group (the heads whose scores fit 128 TMEM columns).  The scores of
// group g + 2 are computed into the buffer group g used, once group g's P V products have
// completed, while the epilogue works on group g + 1.
//
// Biases: one extra K = 16 MMA per GEMM, ones[128 x 16] x bias_tile^T, where the bias tile
// holds the bf16 head and tail of each fp32 bias (columns 0 and 1): D += b_hi + b_lo.
//
// Warp roles: warp 0 issues bulk copies, warp 1 issues tcgen05.mma from one thread (warps 2
// and 3 only complete that warpgroup and hand their registers over), warps 4-11 are the
// epilogue: two warps per TMEM lane quadrant, each owning half of the columns
// (64 of D, i.e. four of the eight heads).  LayerNorm statistics of a row are merged across
// the pair (Welford merge through shared memory, synchronised per quadrant); per-head
// softmax needs no exchange unless a head's keys are split (L_u > 64).  Every wait is
// bounded: a stalled barrier sets an error bit and the kernel unwinds, releasing its tensor
// memory.
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
constexpr int kChunk = 16384;                 // [128 out x 64 in] bf16 weight slice
constexpr int kBiasTile = 4096;               // [128 x 16] bf16 bias tile
// One stream item: a [128 out x 128 in] weight block (two slices) plus its bias tile.  On
// B200 a bulk copy costs about the same time per copy from 16 to 64 KB (a few hundred
// cycles each, copies of one SM largely serialised), so items are as large as the ring
// allows.
constexpr int kSlot = 2 * kChunk + kBiasTile;
constexpr int kStages = 3;
constexpr int kItemsPerLayer = 8;
constexpr int kVecPerLayer = 4 * kD;          // LN1 gain, LN1 shift, LN2 gain, LN2 shift
constexpr int kVecFinal = kD + 4;             // head weight * final LN gain, folded head bias
constexpr int kMaxLpTc = 128;
constexpr int kMaxLayersSmemVec = 5;
constexpr int kEpiThreads = 256;
// Warps 0-3 (one warpgroup): bulk-copy producer, MMA issuer, two idle warps; warps 4-11:
// the epilogue.  The control warpgroup gives registers to the epilogue (setmaxnreg), so
// the epilogue runs without spills: 4 x 32 x kCtlRegs + 8 x 32 x kEpiRegs <= 384 x 168.
constexpr int kThreads = 128 + kEpiThreads;
constexpr int kEpiThread0 = 128;
constexpr int kCtlRegs = 104, kEpiRegs = 200;
static_assert(4 * 32 * kCtlRegs + 8 * 32 * kEpiRegs <= kThreads * 168, "register split exceeds the launch");
constexpr float kQScale = 0.25f * 1.44269504088896341f;  // 1/sqrt(d_h) * log2(e)

// Items: Wq, Wk, Wv, Wo, W1 (output columns 0-127), W1 (128-255), W2 (input rows 0-127),
// W2 (rows 128-255); every item but the first half of W2 carries its GEMM's bias tile.
__host__ __device__ constexpr bool item_has_bias(int j) { return j != 6; }

constexpr int OFF_A = 0;
constexpr int OFF_KV = 32768;                               // 2 x L_p x 128 bf16, L_p <= 128
constexpr int OFF_RING = 98304;
constexpr int OFF_ONES = OFF_RING + kStages * kSlot;        // 204 KB
constexpr int OFF_X = OFF_ONES + kM * 16 * 2;               // [2 slots][2 halves][128] float2
constexpr int OFF_VEC = OFF_X + 2 * 2 * kM * 8;
constexpr int OFF_BAR = OFF_VEC + (kMaxLayersSmemVec * kVecPerLayer + kVecFinal) * 4;
constexpr int SMEM_BYTES = OFF_BAR + 320;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

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
  const uint8_t* wimg;       // [n_layer][kItemsPerLayer][kSlot]
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
  // heads per score group: a group's scores fill at most 128 TMEM columns
  t.hg = t.Lp <= 16 ? 8 : t.Lp <= 32 ? 4 : t.Lp <= 64 ? 2 : 1;
  t.ng = t.Lp == 0 ? 0 : 8 / t.hg;
  return t;
}

// Slot s of head group g holds this head.  The first half of a group's slots are heads of
// the first column half (0-3), the second half heads 4-7, so both epilogue halves get work.
__device__ __forceinline__ int slot_head(int g, int s, int hg) {
  if (hg == 1) return g;
  const int half = hg / 2;
  return s < half ? g * half + s : 4 + g * half + (s - half);
}

// The CTA's mbarriers, 8 bytes apart from one base address (offsets are compile-time, so
// the issuing threads hold one register for all of them).
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t at(int i) const { return base + 8u * (uint32_t)i; }
  __device__ __forceinline__ uint32_t full(int s) const { return at(s); }
  __device__ __forceinline__ uint32_t empty(int s) const { return at(kStages + s); }
  __device__ __forceinline__ uint32_t kv_full() const { return at(2 * kStages); }
  __device__ __forceinline__ uint32_t kv_empty() const { return at(2 * kStages + 1); }
  // MMA -> epilogue
  __device__ __forceinline__ uint32_t ev_qk() const { return at(2 * kStages + 2); }
  __device__ __forceinline__ uint32_t ev_s(int i) const { return at(2 * kStages + 3 + i); }
  __device__ __forceinline__ uint32_t ev_av() const { return at(2 * kStages + 5); }
  __device__ __forceinline__ uint32_t ev_o() const { return at(2 * kStages + 6); }
  __device__ __forceinline__ uint32_t ev_h0() const { return at(2 * kStages + 7); }
  __device__ __forceinline__ uint32_t ev_h1() const { return at(2 * kStages + 8); }
  __device__ __forceinline__ uint32_t ev_y() const { return at(2 * kStages + 9); }
  // epilogue -> MMA
  __device__ __forceinline__ uint32_t e1() const { return at(2 * kStages + 10); }
  __device__ __forceinline__ uint32_t e2() const { return at(2 * kStages + 11); }
  __device__ __forceinline__ uint32_t e3(int i) const { return at(2 * kStages + 12 + i); }
  __device__ __forceinline__ uint32_t e4() const { return at(2 * kStages + 14); }
  __device__ __forceinline__ uint32_t e5() const { return at(2 * kStages + 15); }
  __device__ __forceinline__ uint32_t e6a() const { return at(2 * kStages + 16); }
  __device__ __forceinline__ uint32_t e6b() const { return at(2 * kStages + 17); }
  __device__ __forceinline__ uint32_t drain() const { return at(2 * kStages + 18); }
  __device__ __forceinline__ uint32_t esync() const { return at(2 * kStages + 19); }
  __device__ __forceinline__ uint32_t qsync(int q) const { return at(2 * kStages + 20 + q); }
  // MMA -> MMA: the P V products that read score buffer i have completed
  __device__ __forceinline__ uint32_t av_done(int i) const { return at(2 * kStages + 24 + i); }
};
constexpr int kNumBars = 2 * kStages + 26;
constexpr int kBarBytes = 8 * kNumBars;
static_assert(kBarBytes + 16 <= 320, "barrier area");

// ------------------------------------------------------------------ producer (warp 0, one thread)
template <bool PF>
__device__ void producer(const StackParams& p, uint32_t ring, uint32_t kvbuf, const Bars& b,
                         volatile int* abort_flag) {
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0;
  uint32_t pending = 0, pend_parity = 0;       // bit s: slot s has a copy in flight / its parity
  bool kv_pending = false;
  uint32_t kv_pend_parity = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    for (int l = 0; l < p.n_layer && ok; ++l) {
      const uint8_t* wl = p.wimg + (size_t)l * kItemsPerLayer * kSlot;
      for (int j = 0; j < kItemsPerLayer && ok; ++j) {
        if (!PF && j == 3) {  // the request's K/V images go in between the QKV and O weights
          if (!(ok = mbar_wait(b.kv_empty(), kv_phase ^ 1, abort_flag))) break;
          const uint32_t bytes = 2u * t.Lp * kD * 2u;
          if (bytes) {
            mbar_arrive_expect_tx(b.kv_full(), bytes);
            bulk_g2s(kvbuf, p.req[t.r].kv + (size_t)l * bytes, bytes, b.kv_full());
            kv_pending = true;
            kv_pend_parity = kv_phase;
          } else {
            mbar_arrive(b.kv_full());
          }
          kv_phase ^= 1;
        }
        if (!(ok = mbar_wait(b.empty(stage), phase ^ 1, abort_flag))) break;
        const uint32_t bytes = item_has_bias(j) ? kSlot : 2 * kChunk;
        mbar_arrive_expect_tx(b.full(stage), bytes);
        bulk_g2s(ring + stage * kSlot, wl + (size_t)j * kSlot, bytes, b.full(stage));
        pending |= 1u << stage;
        pend_parity = (pend_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  }
  if (!ok) {  // unwinding: let the copies already issued land before the CTA exits
    for (int s = 0; s < kStages; ++s)
      if ((pending >> s) & 1u)
        for (uint64_t t0 = globaltimer_ns();
             !mbar_try_wait(b.full(s), (pend_parity >> s) & 1u) && globaltimer_ns() - t0 < 200000000ull;) {
        }
    if (kv_pending)
      for (uint64_t t0 = globaltimer_ns();
           !mbar_try_wait(b.kv_full(), kv_pend_parity) && globaltimer_ns() - t0 < 200000000ull;) {
      }
  }
}

// ------------------------------------------------------------------ MMA issuer (warp 1, one thread)
template <bool PF, int HG>
__device__ void mma_issuer(const StackParams& p, uint32_t tmem, uint32_t sA, uint32_t sKV, uint32_t ring,
                           uint32_t sOnes, const Bars& b, volatile int* abort_flag) {
  constexpr uint32_t ID128 = idesc_bf16(kM, 128);
  constexpr uint32_t ID16 = idesc_bf16(kM, 16);
  int stage = 0;
  uint32_t phase = 0, kv_phase = 0;
  uint32_t ph1 = 0, ph2 = 0, ph3a = 0, ph3b = 0, ph4 = 0, ph5 = 0, ph6a = 0, ph6b = 0;
  uint32_t av_pend = 0, av_ph = 0;   // bit i: a P V commit on buffer i not yet waited for / its parity
  bool ok = true;
  auto wait_epi = [&](uint32_t bar, uint32_t& ph) {
    ok = ok && mbar_wait(bar, ph, abort_flag);
    ph ^= 1;
    tc_fence_after();
    return ok;
  };
  // weight block j against the 128-wide K of operand A (shared memory at a_base, or tensor
  // memory columns a_col .. a_col + 63 when A_TMEM); the block's bias tile, if any, last
  auto item = [&](int j, uint32_t a_base, uint32_t dcol, bool acc_first, bool a_tmem) {
    if (!ok) return;
    if (!(ok = mbar_wait(b.full(stage), phase, abort_flag))) return;
    tc_fence_after();
    const uint32_t w = ring + stage * kSlot;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t acc = (kk > 0 || acc_first) ? 1u : 0u;
      if (a_tmem)
        mma_bf16_ta(tmem + dcol, tmem + a_base + kk * 8, sdesc(w + kk * 4096, 2048, 128), ID128, acc);
      else
        mma_bf16(tmem + dcol, sdesc(a_base + kk * 4096, 2048, 128), sdesc(w + kk * 4096, 2048, 128), ID128, acc);
    }
    if (item_has_bias(j)) mma_bf16(tmem + dcol, sdesc(sOnes, 2048, 128), sdesc(w + 2 * kChunk, 2048, 128), ID128, 1u);
    mma_commit(b.empty(stage));
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  };
  for (int tile = blockIdx.x; tile < p.n_tiles && ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    const uint32_t idS = idesc_bf16(kM, t.Lp > 0 ? t.Lp : 16);
    // P V of the last group that used a score buffer must be complete before new scores
    // overwrite its numerators
    auto av_wait = [&](int buf) {
      if (!((av_pend >> buf) & 1u)) return;
      ok = ok && mbar_wait(b.av_done(buf), (av_ph >> buf) & 1u, abort_flag);
      av_ph ^= 1u << buf;
      av_pend &= ~(1u << buf);
      tc_fence_after();
    };
    // scores of head group g into TMEM buffer g % 2
    auto issue_S = [&](int g) {
      const int buf = g & 1;
      av_wait(buf);
      if (!ok) return;
      for (int s = 0; s < HG; ++s) {
        const int h = slot_head(g, s, HG);
        mma_bf16(tmem + 128 + 128 * buf + s * t.Lp, sdesc(sA + h * 4096, 2048, 128),
                 sdesc(sKV + 2 * h * (t.Lp / 8) * 128, (t.Lp / 8) * 128, 128), idS, 0u);
      }
      mma_commit(b.ev_s(buf));
    };
    // O[:, head] += P_head V_head for the heads of group g; P is read from tensor memory
    // (slot s's numerators over the first half of its score columns)
    auto issue_AV = [&](int g) {
      const int buf = g & 1;
      for (int s = 0; s < HG; ++s) {
        const int h = slot_head(g, s, HG);
        const uint32_t pcol = 128 + 128 * buf + s * t.Lp;
        const uint32_t vb = sKV + t.Lp * 256;
        for (int kk = 0; kk < t.Lp / 16; ++kk)
          mma_bf16_ta(tmem + 384 + 16 * h, tmem + pcol + kk * 8, sdesc(vb + (32 * kk + 2 * h) * 128, 2048, 128),
                      ID16, kk > 0 ? 1u : 0u);
      }
      mma_commit(b.av_done(buf));
      av_pend |= 1u << buf;
    };
    for (int l = 0; l < p.n_layer && ok; ++l) {
      // opaque per layer: keeps descriptor arithmetic from being hoisted into registers
      asm volatile("" : "+r"(sA), "+r"(sKV), "+r"(ring), "+r"(sOnes), "+r"(tmem));
      if (!wait_epi(b.e1(), ph1)) break;                // A = LN1(y)
      item(0, sA, 128, false, false);                 // Q + bq
      item(1, sA, 256, false, false);                 // own K + bk
      item(2, sA, 384, false, false);                 // own V + bv
      mma_commit(b.ev_qk());
      if (!wait_epi(b.e2(), ph2)) break;                // A = Q (scaled); own V in registers
      if (!PF) {
        ok = ok && mbar_wait(b.kv_full(), kv_phase, abort_flag);
        kv_phase ^= 1;
        tc_fence_after();
      }
      if (ok && t.ng > 0) issue_S(0);
      if (ok && HG >= 2 && t.ng > 1) issue_S(1);
      if constexpr (HG >= 2) {
        // rounds of gpr groups (the epilogue's GPR); two score buffers are in flight, so
        // after round g0 the scores of groups g0 + 2 .. g0 + 1 + gpr are issued
        constexpr int gpr = 1;
        for (int g0 = 0; g0 < t.ng && ok; g0 += gpr) {
          const bool odd = (g0 / gpr) & 1;
          if (!(odd ? wait_epi(b.e3(1), ph3b) : wait_epi(b.e3(0), ph3a))) break;   // round's numerators written
          for (int gi = 0; gi < gpr; ++gi) issue_AV(g0 + gi);
          for (int gi = 0; gi < gpr; ++gi)
            if (g0 + 2 + gi < t.ng) issue_S(g0 + 2 + gi);
        }
      } else {
        for (int g = 0; g < t.ng && ok; ++g) {
          if (!((g & 1) ? wait_epi(b.e3(1), ph3b) : wait_epi(b.e3(0), ph3a))) break;   // P of group g written
          issue_AV(g);
          // group g + 1 goes to the other score buffer once the P V that last read it is done
          if (g + 1 < t.ng) issue_S(g + 1);
        }
      }
      av_wait(0);
      av_wait(1);
      if (!ok) break;
      if (!PF) mma_commit(b.kv_empty());
      mma_commit(b.ev_av());
      if (!wait_epi(b.e4(), ph4)) break;                // A = attention output
      item(3, sA, 0, true, false);                    // Y += attn Wo + bo
      mma_commit(b.ev_o());
      if (!wait_epi(b.e5(), ph5)) break;                // A = LN2(y)
      item(4, sA, 128, false, false);                 // hidden[0,128) + b1
      mma_commit(b.ev_h0());
      item(5, sA, 256, false, false);                 // hidden[128,256) + b1
      mma_commit(b.ev_h1());
      if (!wait_epi(b.e6a(), ph6a)) break;              // TMEM [384,448) = ReLU(hidden[0,128))
      item(6, 384, 0, true, true);                    // Y += H W2, first half of K
      if (!wait_epi(b.e6b(), ph6b)) break;              // TMEM [448,512) = ReLU(hidden[128,256))
      item(7, 448, 0, true, true);                    // second half of K, + b2
      mma_commit(b.ev_y());
    }
  }
  // drain every MMA still in flight before the tensor memory is released
  mma_commit(b.drain());
  for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.drain(), 0) && globaltimer_ns() - t0 < 500000000ull;) {
  }
}

// ------------------------------------------------------------------ epilogue (warps 2-9)
struct Epi {
  uint32_t trow;        // TMEM address of this row, column 0
  uint32_t rowoff;      // byte offset of this row inside a 128-row core-matrix operand
  int m, hf, q;         // row, column half (0: columns 0-63 / heads 0-3), lane quadrant
  uint32_t sA, sKV, sX;
  const float* vec;     // LayerNorm vectors (shared memory copy when it fits)
  Bars b;
  volatile int* abort_flag;
  bool ok;
  uint32_t ph_qk, ph_s[2], ph_av, ph_o, ph_h0, ph_h1, ph_y, ph_sync, ph_q;

  __device__ bool wait(uint32_t bar, uint32_t& ph) {
    ok = ok && mbar_wait(bar, ph, abort_flag);
    ph ^= 1;
    tc_fence_after();
    return ok;
  }
  __device__ void signal(uint32_t bar) {
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(bar);
  }
  // rendezvous of the 256 epilogue threads (bounded)
  __device__ bool sync() {
    mbar_arrive(b.esync());
    ok = ok && mbar_wait(b.esync(), ph_sync, abort_flag);
    ph_sync ^= 1;
    return ok;
  }
  // exchange one float2 with the other column half of this row through exchange slot
  // `slot`; consecutive exchanges inside one phase must alternate slots
  __device__ float2 swap(float2 mine, int slot) {
    const uint32_t x = sX + slot * (2 * kM * 8);
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(x + (hf * kM + m) * 8), "f"(mine.x), "f"(mine.y)
                 : "memory");
    mbar_arrive(b.qsync(q));
    ok = ok && mbar_wait(b.qsync(q), ph_q, abort_flag);
    ph_q ^= 1;
    float2 o;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(o.x), "=f"(o.y) : "r"(x + ((1 - hf) * kM + m) * 8)
                 : "memory");
    return o;
  }
};

// Compiler-only barrier: keeps the loads of the next step from being hoisted above it, so
// that per-column vectors are not all held in registers at once.
__device__ __forceinline__ void step_barrier() { asm volatile("" ::: "memory"); }

__device__ __forceinline__ void load64(uint32_t taddr, float* v) {
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld16(taddr + c * 16, v + c * 16);
  tmem_wait_ld();
  reg_fence<64>(v);
}

// Row mean / rstd of a 128-wide row held as two 64-column halves (Welford merge).
__device__ __forceinline__ float2 row_stats(Epi& e, const float* y) {
  // four independent partial sums per pass: short dependency chains
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 64; ++i) a[i & 3] += y[i];
  const float mean = ((a[0] + a[1]) + (a[2] + a[3])) * (1.f / 64);
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = 0.f;
#pragma unroll
  for (int i = 0; i < 64; ++i) a[i & 3] = fmaf(y[i] - mean, y[i] - mean, a[i & 3]);
  const float m2 = (a[0] + a[1]) + (a[2] + a[3]);
  const float2 o = e.swap(make_float2(mean, m2), 0);
  const float d = mean - o.x;
  const float mu = 0.5f * (mean + o.x);
  const float var = (m2 + o.y + d * d * 32.f) * (1.f / kD);
  return make_float2(mu, rsqrtf(var + kLnEps));
}

// LayerNorm of this thread's 64 columns -> bf16 into the A operand.
__device__ __forceinline__ void ln_to_A(Epi& e, const float* y, const float* gamma, const float* beta) {
  const float2 st = row_stats(e, y);
  const float4* g4 = reinterpret_cast<const float4*>(gamma + 64 * e.hf);
  const float4* b4 = reinterpret_cast<const float4*>(beta + 64 * e.hf);
#pragma unroll
  for (int kc = 0; kc < 8; ++kc) {
    const float4 ga = g4[2 * kc], gb = g4[2 * kc + 1];
    const float4 ba = b4[2 * kc], bb = b4[2 * kc + 1];
    const float gg[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
    const float bbv[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = fmaf((y[kc * 8 + i] - st.x) * st.y, gg[i], bbv[i]);
    st_row8(e.sA + (8 * e.hf + kc) * 2048 + e.rowoff, v);
    step_barrier();
  }
}

// ReLU of 64 accumulator columns -> bf16 pairs in 32 TMEM columns (an A operand row).
__device__ __forceinline__ void relu_to_tmem(uint32_t tcol, uint32_t dcol) {
  float v[64];
  load64(tcol, v);
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = fmaxf(v[i], 0.f);
  tmem_st_bf16x32(dcol, v);
  tmem_st_bf16x32(dcol + 16, v + 32);
}

template <bool PF, int HG>
__device__ __forceinline__ void epi_tile(const StackParams& p, const TileInfo& t, Epi& e) {
  constexpr int NG = 8 / HG;
  constexpr int SV = HG == 8 ? 16 : HG == 4 ? 32 : 64;   // keys one thread holds for one head
  const int hf = e.hf, m = e.m;
  const uint32_t ycol = e.trow + 64 * hf;
  const float* sd = p.domain_emb + (size_t)p.req[t.r].domain * kD + 64 * hf;
  // ---- Y = t + s_d (rows past the request's end are zero and never stored)
  {
    float y[64];
    const float4* sd4 = reinterpret_cast<const float4*>(sd);
    const bool live = m < t.rows;
    if (PF) {
      const float4* src = reinterpret_cast<const float4*>(p.utokens + (t.row0 + m) * kD + 64 * hf);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 u = live ? __ldg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 d = __ldg(sd4 + c);
        y[4 * c] = live ? u.x + d.x : 0.f;
        y[4 * c + 1] = live ? u.y + d.y : 0.f;
        y[4 * c + 2] = live ? u.z + d.z : 0.f;
        y[4 * c + 3] = live ? u.w + d.w : 0.f;
        step_barrier();
      }
    } else {
      const uint4* src = reinterpret_cast<const uint4*>(p.tokens + (t.row0 + m) * kD + 64 * hf);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 u = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        const float4 da = __ldg(sd4 + 2 * c), db = __ldg(sd4 + 2 * c + 1);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const float d[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          y[c * 8 + 2 * i] = live ? __uint_as_float(w[i] << 16) + d[2 * i] : 0.f;
          y[c * 8 + 2 * i + 1] = live ? __uint_as_float(w[i] & 0xFFFF0000u) + d[2 * i + 1] : 0.f;
        }
        step_barrier();
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_st16(ycol + 16 * c, y + 16 * c);
    tmem_wait_st();
  }

  for (int l = 0; l < p.n_layer; ++l) {
    const float* vl = e.vec + (size_t)l * kVecPerLayer;
    // ---- LN1 -> A
    if (l > 0 && !e.wait(e.b.ev_y(), e.ph_y)) return;
    {
      float y[64];
      load64(ycol, y);
      ln_to_A(e, y, vl, vl + kD);
    }
    e.signal(e.b.e1());
    // ---- Q (scaled) -> A; own score per head; own V -> registers; user side: K/V images
    if (!e.wait(e.b.ev_qk(), e.ph_qk)) return;
    if (PF) {
      if (threadIdx.x == kEpiThread0 && l > 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
      if (!e.sync()) return;                       // the K/V images are free to overwrite
    }
    float sself[4];
    uint32_t vself[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int h = 4 * hf + j;
      float qv[16], kv[16], vv[16];
      tmem_ld16(e.trow + 128 + 16 * h, qv);
      tmem_ld16(e.trow + 256 + 16 * h, kv);
      tmem_ld16(e.trow + 384 + 16 * h, vv);
      tmem_wait_ld();
      reg_fence<16>(qv);
      reg_fence<16>(kv);
      reg_fence<16>(vv);
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        qv[i] *= kQScale;
        s = fmaf(qv[i], kv[i], s);
      }
      sself[j] = PF ? -INFINITY : s;
#pragma unroll
      for (int i = 0; i < 8; ++i) vself[j][i] = pack2(vv[2 * i], vv[2 * i + 1]);
      st_row8(e.sA + (2 * h) * 2048 + e.rowoff, qv);
      st_row8(e.sA + (2 * h + 1) * 2048 + e.rowoff, qv + 8);
      if (PF && m < t.Lp) {
        // K image row m, V^T image column m (zero past L_u)
        const bool live = m < t.L_u;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          kv[i] = live ? kv[i] : 0.f;
          vv[i] = live ? vv[i] : 0.f;
        }
        const uint32_t kb = e.sKV + (m >> 3) * 128 + (m & 7) * 16;
        st_row8(kb + (2 * h) * (t.Lp / 8) * 128, kv);
        st_row8(kb + (2 * h + 1) * (t.Lp / 8) * 128, kv + 8);
        const uint32_t vb = e.sKV + t.Lp * 256 + (m >> 3) * 2048 + (m & 7) * 2;
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
    if (PF) {  // store this layer's K/V images to the cache with one bulk copy
      fence_proxy_async_smem();
      if (!e.sync()) return;
      if (threadIdx.x == kEpiThread0) {
        const uint32_t bytes = 2u * t.Lp * kD * 2u;
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(p.kv_out + (size_t)l * bytes),
                     "r"(e.sKV), "r"(bytes)
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    e.signal(e.b.e2());
    // ---- softmax over [user keys of the request, own key], one head group at a time
    float pself[4] = {1.f, 1.f, 1.f, 1.f}, linv[4] = {1.f, 1.f, 1.f, 1.f};
    if constexpr (HG >= 2) {
      // One score group per round: while the epilogue works on group g + 1 the tensor core
      // multiplies group g's numerators by V and computes group g + 2's scores into the
      // buffer group g used.  (Two groups per round measured no faster: it loses that
      // overlap.)  Rounds signal e3(0) and e3(1) in turn, so the MMA thread's wait on one
      // never sees it complete twice.
      constexpr int GPR = 1;
      const int nb = t.Lp / 16;                   // 16-key blocks holding keys (>= 1)
      const int tail = t.L_u - 16 * (nb - 1);     // keys in the last block (1..16)
#pragma unroll
      for (int g0 = 0; g0 < NG; g0 += GPR) {
        if (g0 >= t.ng) break;
#pragma unroll
        for (int gi = 0; gi < GPR; ++gi)
          if (!e.wait(e.b.ev_s((g0 + gi) & 1), e.ph_s[(g0 + gi) & 1])) return;
#pragma unroll
        for (int gi = 0; gi < GPR; ++gi) {
          const int g = g0 + gi;
          const uint32_t sbuf = e.trow + 128 + 128 * (g & 1);
#pragma unroll
          for (int j = 0; j < HG / 2; ++j) {
            const int jj = g * (HG / 2) + j;        // this half's head index (0..3)
            const int slot = hf * (HG / 2) + j;
            float sv[SV];
#pragma unroll
            for (int c = 0; c < SV / 16; ++c) {
              if (c < nb) {
                tmem_ld16(sbuf + slot * t.Lp + 16 * c, sv + 16 * c);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[16 * c + i] = -INFINITY;
              }
            }
            tmem_wait_ld();
            reg_fence<SV>(sv);
            // padding keys (L_u not a multiple of 16) -> -inf, so the loops below need no masks
            if (tail < 16) {
#pragma unroll
              for (int i = 0; i < SV; ++i) sv[i] = i < t.L_u ? sv[i] : -INFINITY;
            }
            // max: four chains of three-input maxima
            float m4[4] = {sself[jj], -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < SV; i += 8) {
              m4[0] = max3(m4[0], sv[i], sv[i + 1]);
              m4[1] = max3(m4[1], sv[i + 2], sv[i + 3]);
              m4[2] = max3(m4[2], sv[i + 4], sv[i + 5]);
              m4[3] = max3(m4[3], sv[i + 6], sv[i + 7]);
            }
            const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            // exponentials; the subtraction and the running sums on packed pairs
            const uint64_t neg = f32x2(-mx, -mx);
            uint64_t acc[2] = {f32x2(0.f, 0.f), f32x2(0.f, 0.f)};
#pragma unroll
            for (int i = 0; i < SV; i += 2) {
              float x0, x1;
              f32x2_split(add_f32x2(f32x2(sv[i], sv[i + 1]), neg), x0, x1);
              sv[i] = ex2(x0);
              sv[i + 1] = ex2(x1);
              acc[(i >> 1) & 1] = add_f32x2(acc[(i >> 1) & 1], f32x2(sv[i], sv[i + 1]));
            }
            float a0, a1, b0, b1;
            f32x2_split(acc[0], a0, a1);
            f32x2_split(acc[1], b0, b1);
            const float sum = (a0 + a1) + (b0 + b1);
            // numerators as bf16 over the first half of this slot's own score columns (the
            // P V products read only the first L_p / 2 of them)
            const uint32_t pcol = sbuf + slot * t.Lp;
            if constexpr (SV == 16) {
              tmem_st_bf16x16(pcol, sv);
            } else {
#pragma unroll
              for (int c = 0; c < SV / 32; ++c) tmem_st_bf16x32(pcol + 16 * c, sv + 32 * c);
            }
            pself[jj] = ex2(sself[jj] - mx);
            linv[jj] = 1.f / (sum + pself[jj]);
          }
        }
        e.signal(e.b.e3((g0 / GPR) & 1));
      }
    } else {
      // L_u > 64: one head per group, its keys split between the two column halves
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        if (!e.wait(e.b.ev_s(g & 1), e.ph_s[g & 1])) return;
        const uint32_t sbuf = e.trow + 128 + 128 * (g & 1);
        const int k0 = 64 * hf;
        const int nk = min(64, t.Lp - k0);       // > 0: Lp >= 80
        float sv[64];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < nk / 16) tmem_ld16(sbuf + k0 + 16 * c, sv + 16 * c);
        tmem_wait_ld();
        reg_fence<64>(sv);
        const bool owner = (g >> 2) == hf;       // this half owns head g (and its own score)
        float m4[4] = {owner ? sself[g & 3] : -INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < nk && k0 + i < t.L_u) m4[i & 3] = fmaxf(m4[i & 3], sv[i]);
        float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        mx = fmaxf(mx, e.swap(make_float2(mx, 0.f), 0).x);
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float ev = (i < nk && k0 + i < t.L_u) ? ex2(sv[i] - mx) : 0.f;
          sv[i] = ev;
          s4[i & 3] += ev;
        }
        const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        // keys 64 hf .. as bf16 from column 32 hf of the buffer: over this half's own scores
        // (hf = 0) or the first half's, which both halves have read before the max exchange
        tmem_st_bf16x32(sbuf + 32 * hf, sv);
        tmem_st_bf16x32(sbuf + 32 * hf + 16, sv + 32);
        const float ps = owner ? ex2(sself[g & 3] - mx) : 0.f;
        const float tot = sum + ps + e.swap(make_float2(sum + ps, 0.f), 1).x;
        if (owner) {
          pself[g & 3] = ps;
          linv[g & 3] = 1.f / tot;
        }
        e.signal(e.b.e3(g & 1));
      }
    }
    // ---- attention output = (sum_j p_j v_j + p_self v_self) / l  -> A
    if (!e.wait(e.b.ev_av(), e.ph_av)) return;
    const bool has_users = t.ng > 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int h = 4 * hf + j;
      float o[16];
      tmem_ld16(e.trow + 384 + 16 * h, o);
      tmem_wait_ld();
      reg_fence<16>(o);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t w = vself[j][i];
        const float v0 = __uint_as_float(w << 16), v1 = __uint_as_float(w & 0xFFFF0000u);
        o[2 * i] = ((has_users ? o[2 * i] : 0.f) + pself[j] * v0) * linv[j];
        o[2 * i + 1] = ((has_users ? o[2 * i + 1] : 0.f) + pself[j] * v1) * linv[j];
      }
      st_row8(e.sA + (2 * h) * 2048 + e.rowoff, o);
      st_row8(e.sA + (2 * h + 1) * 2048 + e.rowoff, o + 8);
    }
    e.signal(e.b.e4());
    // ---- LN2 -> A
    if (!e.wait(e.b.ev_o(), e.ph_o)) return;
    {
      float y[64];
      load64(ycol, y);
      ln_to_A(e, y, vl + 2 * kD, vl + 3 * kD);
    }
    e.signal(e.b.e5());
    // ---- ReLU(hidden) -> P0 (first half of the hidden units) and A (second half)
    if (!e.wait(e.b.ev_h0(), e.ph_h0)) return;
    relu_to_tmem(e.trow + 128 + 64 * hf, e.trow + 384 + 32 * hf);
    e.signal(e.b.e6a());
    if (!e.wait(e.b.ev_h1(), e.ph_h1)) return;
    relu_to_tmem(e.trow + 256 + 64 * hf, e.trow + 448 + 32 * hf);
    e.signal(e.b.e6b());
  }
  // ---- head: w . LN_f(y) + b
  if (!e.wait(e.b.ev_y(), e.ph_y)) return;
  if (PF) return;
  float y[64];
  load64(ycol, y);
  const float2 st = row_stats(e, y);
  const float* vf = e.vec + (size_t)p.n_layer * kVecPerLayer;
  const float4* w4 = reinterpret_cast<const float4*>(vf + 64 * hf);
  float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 w = w4[i];
    a4[0] = fmaf((y[4 * i] - st.x) * st.y, w.x, a4[0]);
    a4[1] = fmaf((y[4 * i + 1] - st.x) * st.y, w.y, a4[1]);
    a4[2] = fmaf((y[4 * i + 2] - st.x) * st.y, w.z, a4[2]);
    a4[3] = fmaf((y[4 * i + 3] - st.x) * st.y, w.w, a4[3]);
    step_barrier();
  }
  const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
  const float tot = acc + e.swap(make_float2(acc, 0.f), 1).x;
  if (hf == 0 && m < t.rows) p.scores[t.row0 + m] = tot + vf[kD];
}

template <bool PF, int HG>
__device__ void epilogue(const StackParams& p, uint32_t tmem, uint32_t sA, uint32_t sKV,
                         uint32_t sX, uint32_t sOnes, float* svec, const Bars& b, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Epi e;
  e.q = warp & 3;
  e.m = e.q * 32 + lane;
  e.hf = (warp - 4) >> 2;
  e.trow = tmem + ((uint32_t)(e.q * 32) << 16);
  e.rowoff = (e.m >> 3) * 128 + (e.m & 7) * 16;
  e.sA = sA;
  e.sKV = sKV;
  e.sX = sX;
  e.b = b;
  e.abort_flag = abort_flag;
  e.ok = true;
  e.ph_qk = e.ph_s[0] = e.ph_s[1] = e.ph_av = e.ph_o = e.ph_h0 = e.ph_h1 = e.ph_y = e.ph_sync = e.ph_q = 0;
  // the constant ones tile: columns 0 and 1 of every row are 1 (bias head and tail)
  if (e.hf == 0) {
    const float one2[8] = {1.f, 1.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, zero[8] = {};
    st_row8(sOnes + e.rowoff, one2);
    st_row8(sOnes + 2048 + e.rowoff, zero);
  }
  // LayerNorm vectors and the head weight: a shared-memory copy when they fit
  const int nvec = p.n_layer * kVecPerLayer + kVecFinal;
  if (p.n_layer <= kMaxLayersSmemVec) {
    const int tid = threadIdx.x - kEpiThread0;
    for (int i = tid; i < nvec; i += kEpiThreads) svec[i] = __ldg(p.vec + i);
    if (!e.sync()) return;
    e.vec = svec;
  } else {
    e.vec = p.vec;
  }
  for (int tile = blockIdx.x; tile < p.n_tiles && e.ok; tile += gridDim.x) {
    const TileInfo t = tile_info(p, tile);
    epi_tile<PF, HG>(p, t, e);   // the host launches one kernel per head-group size
  }
}

template <bool PF, int HG>
__global__ void __launch_bounds__(kThreads, 1) stack_kernel(const __grid_constant__ StackParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t sA = base + OFF_A, sKV = base + OFF_KV, ring = base + OFF_RING;
  const uint32_t sOnes = base + OFF_ONES, sX = base + OFF_X;
  float* svec = reinterpret_cast<float*>(smem + OFF_VEC);
  const Bars b{base + OFF_BAR};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + kBarBytes);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + kBarBytes + 8);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(b.full(s), 1);
      mbar_init(b.empty(s), 1);
    }
    mbar_init(b.kv_full(), 1);
    mbar_init(b.kv_empty(), 1);
    for (uint32_t a : {b.ev_qk(), b.ev_s(0), b.ev_s(1), b.ev_av(), b.ev_o(), b.ev_h0(), b.ev_h1(), b.ev_y(), b.drain(),
                       b.av_done(0), b.av_done(1)})
      mbar_init(a, 1);
    for (uint32_t a : {b.e1(), b.e2(), b.e3(0), b.e3(1), b.e4(), b.e5(), b.e6a(), b.e6b(), b.esync()}) mbar_init(a, kEpiThreads);
    for (int q = 0; q < 4; ++q) mbar_init(b.qsync(q), 64);
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

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));
    if (warp == 0 && lane == 0) producer<PF>(p, ring, sKV, b, abort_flag);
    if (warp == 1 && lane == 0) mma_issuer<PF, HG>(p, tmem, sA, sKV, ring, sOnes, b, abort_flag);
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
    epilogue<PF, HG>(p, tmem, sA, sKV, sX, sOnes, svec, b, abort_flag);
    if (PF && threadIdx.x == kEpiThread0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, STATUS_KERNEL_TIMEOUT);
}

// ------------------------------------------------------------------ host: operand images

uint16_t bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;  // round to nearest even
  return (uint16_t)u;
}
float bf16_value(uint16_t h) {
  const uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// W^T slice [n0, n0+128) x [k0, k0+64) of W [K][N] (row-major, W[k][n]) in core-matrix layout.
void put_chunk(uint16_t* dst, const float* W, int N, int n0, int k0) {
  for (int n = 0; n < 128; ++n)
    for (int k = 0; k < 64; ++k)
      dst[((size_t)(k / 8) * 16 + n / 8) * 64 + (n % 8) * 8 + (k % 8)] = bf16_bits(W[(size_t)(k0 + k) * N + n0 + n]);
}

// Bias tile [128 x 16]: column 0 the bf16 nearest to b[n0+n], column 1 the bf16 of the rest.
void put_bias(uint16_t* dst, const float* bias, int n0) {
  for (int n = 0; n < 128; ++n) {
    const float v = bias[n0 + n];
    const uint16_t hi = bf16_bits(v);
    const uint16_t lo = bf16_bits(v - bf16_value(hi));
    for (int k = 0; k < 16; ++k)
      dst[((size_t)(k / 8) * 16 + n / 8) * 64 + (n % 8) * 8 + (k % 8)] = k == 0 ? hi : k == 1 ? lo : 0;
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
  const size_t se = kSlot / 2;  // elements per stream slot
  std::vector<uint16_t> img((size_t)N * kItemsPerLayer * se, 0);
  std::vector<float> vec((size_t)N * kVecPerLayer + kVecFinal, 0.f);
  for (int l = 0; l < N; ++l) {
    // weights go in unchanged (exact bf16 values); LayerNorm gains/shifts stay fp32 in the
    // epilogue; biases become bias tiles next to the last slice of their GEMM
    const tr_layer_weights& L = w->layers[l];
    uint16_t* li = img.data() + (size_t)l * kItemsPerLayer * se;
    // item j: slice (K 0-63) | slice (K 64-127) | bias tile
    auto half = [&](int j, int h) { return li + (size_t)j * se + (size_t)h * (kChunk / 2); };
    auto bias = [&](int j) { return li + (size_t)j * se + kChunk; };
    const float* Wn[4] = {L.Wq, L.Wk, L.Wv, L.Wo};
    const float* bn[4] = {L.bq, L.bk, L.bv, L.bo};
    for (int j = 0; j < 4; ++j) {
      put_chunk(half(j, 0), Wn[j], D, 0, 0);
      put_chunk(half(j, 1), Wn[j], D, 0, 64);
      put_bias(bias(j), bn[j], 0);
    }
    for (int j = 0; j < 2; ++j) {   // W1, output columns 128 j .. 128 j + 127
      put_chunk(half(4 + j, 0), L.W1, H, 128 * j, 0);
      put_chunk(half(4 + j, 1), L.W1, H, 128 * j, 64);
      put_bias(bias(4 + j), L.b1, 128 * j);
    }
    for (int q = 0; q < 4; ++q) put_chunk(half(6 + q / 2, q % 2), L.W2, D, 0, 64 * q);
    put_bias(bias(7), L.b2, 0);
    float* v = vec.data() + (size_t)l * kVecPerLayer;
    for (int j = 0; j < D; ++j) {
      v[j] = L.ln1_g[j];
      v[D + j] = L.ln1_b[j];
      v[2 * D + j] = L.ln2_g[j];
      v[3 * D + j] = L.ln2_b[j];
    }
  }
  float* vf = vec.data() + (size_t)N * kVecPerLayer;
  double bh = w->b_head;
  for (int j = 0; j < D; ++j) {
    vf[j] = (float)((double)w->w_head[j] * w->lnf_g[j]);
    bh += (double)w->w_head[j] * w->lnf_b[j];
  }
  vf[D] = (float)bh;
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
  m->tc_stack_layer_bytes = (size_t)kItemsPerLayer * kSlot;
  m->tc_vec = reinterpret_cast<const float*>((uint8_t*)m->tc_blob + img_bytes);
  m->tc_vec_layer_floats = kVecPerLayer;
  return TR_OK;
}

int hg_of(int L_u) {
  const int Lp = (L_u + 15) & ~15;
  return Lp <= 16 ? 8 : Lp <= 32 ? 4 : Lp <= 64 ? 2 : 1;
}

template <bool PF>
tr_status launch_stack(int hg, int grid, const StackParams& p, cudaStream_t st) {
  void (*k)(StackParams) = hg == 8 ? stack_kernel<PF, 8> : hg == 4 ? stack_kernel<PF, 4>
                         : hg == 2 ? stack_kernel<PF, 2> : stack_kernel<PF, 1>;
  TR_TRY(ensure_smem_attr((const void*)k, SMEM_BYTES));
  k<<<grid, kThreads, SMEM_BYTES, st>>>(p);
  TR_LAUNCH_CHECK(PF ? "stack_kernel (user side)" : "stack_kernel");
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
  if ((uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "tokens not 16-byte aligned");
  for (int r = 0; r < R; ++r)
    if ((uintptr_t)kv[r] % 16 && L_u[r] > 0 && req_offsets[r + 1] > req_offsets[r])
      return fail(TR_ERR_INVALID_ARG, "kv[%d] is not 16-byte aligned", r);
  int sms = 148, dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  // one launch per head-group size (requests of one class share the kernel's code path)
  for (int hg : {2, 1, 4, 8}) {
    StackParams p{};
    p.tokens = static_cast<const __nv_bfloat16*>(tokens);
    p.scores = scores;
    p.wimg = static_cast<const uint8_t*>(m->tc_stack);
    p.vec = m->tc_vec;
    p.domain_emb = m->domain_emb;
    p.status = ds->status;
    p.n_layer = m->desc.n_layer;
    int tiles = 0, k = 0;
    for (int r = 0; r < R; ++r) {
      const int64_t nr = req_offsets[r + 1] - req_offsets[r];
      if (hg_of(L_u[r]) != hg || nr == 0) continue;
      p.req[k].kv = static_cast<const uint8_t*>(kv[r]);
      p.req[k].cand_off = req_offsets[r];
      p.req[k].n = nr;
      p.req[k].tile_off = tiles;
      p.req[k].L_u = L_u[r];
      p.req[k].domain = domain[r];
      tiles += (int)((nr + kM - 1) / kM);
      ++k;
    }
    if (tiles == 0) continue;
    p.R = k;
    p.n_tiles = tiles;
    TR_TRY(launch_stack<false>(hg, std::min(tiles, sms), p, st));
  }
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
  return launch_stack<true>(hg_of(L_u), 1, p, st);
}

}  // namespace tr
