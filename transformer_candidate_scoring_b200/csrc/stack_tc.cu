// Fused Transformer stack on tcgen05 tensor cores (TransRetrieval §3.3, §3.4, deployment
// section "Hardware-aware inference optimization"), for D = 64 and D = 128 (d_h = 16, FFN
// hidden 2D).  One kernel serves both sides of a request:
//   score mode  candidate tiles: every row attends to its request's cached user K/V plus its
//               own key/value; final LayerNorm and the linear head give the score;
//   user mode   the request's user tokens as one tile, attending to each other; each layer's
//               K/V images are written to the request's cache (one bulk store per layer).
//
// Two 128-row tiles ("slots") are in flight per CTA, so that one slot's LayerNorm, softmax
// and hand-offs run while the tensor core works on the other slot's products.  Each slot
// owns 256 TMEM columns, 4 P epilogue warps (P threads per tile row: two at D = 128, each
// with half of the row's columns and every other head, one at D = 64) and an MMA-issuing
// thread; the two slots of a CTA take two consecutive tiles of one request (a "unit") and
// share its K/V images and every weight item of the stream.
//
//   TMEM (per slot, 256 fp32 columns, lane = tile row)
//     [0, D)        Y, the residual stream; the O and FFN2 products (and their biases)
//                   accumulate into it in place
//     [D, D + 128)  work area W, in turn: own K, own V, Q (each read out by the epilogue),
//                   the scores of one head group (numerators written back over them as
//                   fp16, the A operand of P V, whose result lands beside them; with one
//                   epilogue thread per row also of a product with ones that gives the
//                   numerators' row sum, which two threads per row add up themselves), the
//                   FFN hidden units (a 128-wide half at a time; ReLU written back as fp16,
//                   the A operand of W2)
//   shared memory
//     A      per slot [128 x D] fp16: LN1 output -> Q -> attention output -> LN2 output
//     KV     the unit's K and V^T images of the current layer (score mode: loaded by bulk
//            copy; user mode: written by the epilogue, then stored to the cache)
//     ring   weight items in consumption order (K, V, Q, O, W1, W2 per layer), each
//            consumed by both slots before its buffer is refilled
//     ones   the [128 x 16] A operand that turns a bias tile into "+ bias" in one MMA
//     vec    LayerNorm gains/shifts of every layer and the folded head weight
//
// Operands are fp16 (the weights are bf16 values, converted exactly; activations are
// rounded to fp16, whose 11-bit significand keeps the error of the five-layer stack a few
// times below that of bf16 operands at the same tensor-core rate); accumulation, LayerNorm
// and softmax are fp32.  A model whose parameters could push an fp16 operand out of range
// is not built for this kernel (it runs on the CUDA-core path).
//
// Warp roles: warp 0 streams weight items, warp 3 streams K/V images (and owns the TMEM
// allocation), warps 1 and 2 issue the MMAs of slot 0 and slot 1, the next 4 P warps are the
// epilogue of slot 0 and the last 4 P that of slot 1.  Every epilogue/MMA hand-off of a slot is a strict
// alternation on two mbarriers.  Every wait is bounded: a stalled barrier sets an error bit
// and the kernel unwinds, releasing its tensor memory.
#include <cuda_fp16.h>
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

constexpr int kM = 128;
constexpr int kSlotCols = 256;
constexpr int kWork = 128;
// Epilogue threads per tile row (P): two at D = 128, where a row's epilogue work is large
// enough to split, one at D = 64.  The launch has a control warpgroup and 4 P epilogue
// warps per slot; `setmaxnreg` moves registers from the control warps to the epilogues.
template <int D>
struct Par {
  static constexpr int P = D == 128 ? 2 : 1;
  static constexpr int kSlotThreads = 128 * P;
  static constexpr int kThreads = 128 + 2 * kSlotThreads;
  static constexpr int kLaunchRegs = P == 2 ? 96 : 168;   // 65,536 / kThreads, rounded down to 8
  static constexpr int kCtlRegs = P == 2 ? 40 : 56, kEpiRegs = P == 2 ? 104 : 224;
  static_assert(4 * 32 * kCtlRegs + 2 * kSlotThreads * kEpiRegs <= kThreads * kLaunchRegs,
                "register split exceeds the launch");
  static_assert(kThreads * kLaunchRegs <= 65536, "launch registers");
};
constexpr int kMaxParts = 2;
constexpr int kMaxStages = 4;
constexpr int kMaxLp = 128;
constexpr float kL2E = 1.44269504088896341f;
constexpr int kSmemLimit = 232448;
// The constant operands: the [128 x 16] A tile whose columns 0 and 1 are ones (bias
// products), then at kOnesBOff a [16 x 16] B tile of ones (row sums of the numerators).
constexpr int kOnesBOff = kM * 16 * 2;
constexpr int kOnesBytes = kOnesBOff + 1024;

// fp16 x fp16 -> fp32, both operands K-major
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// One GEMM of the weight stream: its B operand [N x K] (core-matrix layout, K-major) at
// byte `off` of weight item `item`, and its [N x 16] bias tile at byte `bias` (-1: none).
struct Piece {
  int item, off, N, K, bias;
};
enum { P_K = 0, P_V = 1, P_Q = 2, P_O = 3, P_W1A = 4, P_W2A = 5, P_W1B = 6, P_W2B = 7 };

template <int D>
struct Cfg;
// D = 128: one item per GEMM: K, V, Q, O, W1 (hidden 0-127), W2 (hidden 0-127, no bias),
// W1 (hidden 128-255), W2 (hidden 128-255, + b2).  32 KB of weights + a 4 KB bias tile.
template <>
struct Cfg<128> {
  static constexpr int kNH = 8, kItems = 8, kPieces = 8, kItemBytes = 36864, kFfnHalves = 2;
  __host__ __device__ static constexpr Piece piece(int p) { return Piece{p, 0, 128, 128, p == P_W2A ? -1 : 32768}; }
  __host__ __device__ static constexpr int item_bytes(int j) { return j == P_W2A ? 32768 : 36864; }
};
// D = 64: two items per layer: [K | V | Q | O] (8 KB + a 2 KB bias tile each) and
// [W1 (N = 128) + bias | W2 (K = 128) + bias].
template <>
struct Cfg<64> {
  static constexpr int kNH = 4, kItems = 2, kPieces = 6, kItemBytes = 40960, kFfnHalves = 1;
  __host__ __device__ static constexpr Piece piece(int p) {
    return p < 4 ? Piece{0, p * 10240, 64, 64, p * 10240 + 8192}
                 : (p == P_W1A ? Piece{1, 0, 128, 64, 16384} : Piece{1, 20480, 64, 128, 36864});
  }
  __host__ __device__ static constexpr int item_bytes(int j) { return j == 0 ? 40960 : 38912; }
};

// The LayerNorm gains and shifts are folded into the weights and biases of the products
// that follow them (K, V, Q after LN1; W1 after LN2): LN(y) W + b = z (g o W) + (beta W + b),
// z the standardized row.  The epilogue only standardizes; the one vector it still reads is
// the head's (w o g_f and the folded bias).
template <int D>
constexpr int vec_floats() { return D + 4; }

// Head groups of one launch: SW (32, 64 or 128) is at least the launch's longest padded user
// sequence.  A head owns HW = max(SW, 64) work-area columns: its scores (Lp columns), then,
// written over them, its numerators as fp16 pairs (Lp / 2 columns), and from column HW / 2
// the P V product (16 columns) and the numerators' row sum (16 equal columns).  A group is
// the HG heads that fit.
template <int D, int SW>
struct Groups {
  static constexpr int HW = SW < 64 ? 64 : SW;
  static constexpr int HG = kWork / HW;
  static constexpr int NG = Cfg<D>::kNH / HG;
  static_assert(SW == 32 || SW == 64 || SW == 128, "head slot width");
};

struct ReqInfo {
  const uint8_t* kv;          // score mode: the request's K/V images; user mode: the cache to write
  const float* utokens;       // user mode: fp32 user tokens [L_u][D]
  long long cand_off;
  long long n;                // candidates (score mode) / user tokens (user mode)
  int unit_off;
  int L_u;
  int domain;
  int n_pair;                 // the request's first n_pair units hold two tiles, the rest one
};

struct StackParams {
  const float* tokens;        // score mode: fp32 candidate tokens [n][D]
  const uint16_t* tokens_h;   // candidates of lt tokens: bf16 tokens [n * lt][D]
  int lt;                     // tokens per candidate (1: one compressed token each)
  float* scores;
  const uint8_t* wimg;        // [n_layer][kItems][kItemBytes]
  const float* vec;           // [n_layer][4 D] + [D + 4]
  const float* domain_emb;    // fp32 [n_domains][D]
  int* status;
  int n_layer, n_units, R, pair;
  int off_kv, off_ring, off_ones, off_xch, off_vec, off_bar, stages;
  // where slot 0 lets slot 1 start a unit of two tiles (layer 0): 0 after its own-V phase,
  // 1 after the attention of its second head group.  Slot 0 alone may run at most `stages`
  // weight items ahead, so with a two-item ring the gate must open before it needs Q.
  int gate_phase;
  ReqInfo req[TR_MAX_REQUESTS];
};

struct Tile {
  bool active;
  int r, rows, L_u, Lp, dom;
  long long row0;
};

template <int D>
__device__ __forceinline__ Tile tile_of(const StackParams& p, int u, int slot) {
  int r = 0;
  while (r + 1 < p.R && u >= p.req[r + 1].unit_off) ++r;
  Tile t;
  t.r = r;
  const int k = u - p.req[r].unit_off, np = p.req[r].n_pair;
  const bool two = p.pair && k < np;
  const long long local = two ? 2ll * k + slot : (long long)np + k;   // np pair units, then singles
  t.row0 = p.req[r].cand_off + local * kM;
  const long long end = p.req[r].cand_off + p.req[r].n;
  t.active = (slot == 0 || two) && t.row0 < end;
  t.rows = t.active ? (int)min((long long)kM, end - t.row0) : 0;
  t.L_u = p.req[r].L_u;
  t.Lp = (t.L_u + 15) & ~15;
  t.dom = p.req[r].domain;
  return t;
}

// The CTA's mbarriers, 8 bytes apart.
struct Bars {
  uint32_t base;
  __device__ __forceinline__ uint32_t at(int i) const { return base + 8u * (uint32_t)i; }
  __device__ __forceinline__ uint32_t full(int s) const { return at(s); }
  __device__ __forceinline__ uint32_t empty(int s) const { return at(kMaxStages + s); }
  __device__ __forceinline__ uint32_t kv_full() const { return at(2 * kMaxStages); }
  __device__ __forceinline__ uint32_t kv_empty(int slot) const { return at(2 * kMaxStages + 1 + slot); }
  __device__ __forceinline__ uint32_t e2m(int slot) const { return at(2 * kMaxStages + 3 + slot); }
  __device__ __forceinline__ uint32_t m2e(int slot) const { return at(2 * kMaxStages + 5 + slot); }
  __device__ __forceinline__ uint32_t mm(int slot) const { return at(2 * kMaxStages + 7 + slot); }
  __device__ __forceinline__ uint32_t drain(int slot) const { return at(2 * kMaxStages + 9 + slot); }
  // epilogue turn of slot s (passed between the two slots of a unit)
  __device__ __forceinline__ uint32_t tok(int slot) const { return at(2 * kMaxStages + 11 + slot); }
  // the exchange between the two parts of the rows of lane quadrant q of slot s
  __device__ __forceinline__ uint32_t xch(int slot, int q) const { return at(2 * kMaxStages + 13 + 4 * slot + q); }
};
constexpr int kNumBars = 2 * kMaxStages + 21;
constexpr int kXchBytes = 2 * kMaxParts * kM * 8;   // per slot: two alternating float2 buffers
constexpr int kBarArea = 8 * kNumBars + 32;   // + TMEM address and abort flag

// ------------------------------------------------------------------ small helpers
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float h_lo(uint32_t w) { return __low2float(*reinterpret_cast<const __half2*>(&w)); }
__device__ __forceinline__ float h_hi(uint32_t w) { return __high2float(*reinterpret_cast<const __half2*>(&w)); }
// eight fp32 values -> one 16-byte row of a core matrix (fp16)
__device__ __forceinline__ void st_row8h(uint32_t addr, const float* v) {
  st_shared_v4(addr, pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
}
__device__ __forceinline__ void ld8(const float* p, float* o) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  tmem_ld16(taddr, v);
  tmem_ld16(taddr + 16, v + 16);
}
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return __uint_as_float(r);
}
__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Softmax numerators two at a time: the exponents x (fp32, already shifted by the row
// maximum, so x <= 0) are rounded to an fp16 pair and raised by one packed 2^x, giving the
// fp16 numerators that the P V product consumes.  -inf (a masked key) gives 0.  Every path and slot width computes a key this way, so that a candidate's score
// does not depend on the other requests of its launch.
__device__ __forceinline__ uint32_t exp2_h2(float a, float b) {   // a -> low half
  uint32_t h, r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(b), "f"(a));
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(r) : "r"(h));
  return r;
}
// s_lo += low half of w, s_hi += high half (fp16 -> fp32 adds)
__device__ __forceinline__ void acc_h2(float& s_lo, float& s_hi, uint32_t w) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "add.rn.f32.f16 %0, l, %0;\n\tadd.rn.f32.f16 %1, h, %1;\n\t}"
      : "+f"(s_lo), "+f"(s_hi)
      : "r"(w));
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Bounded wait of one thread for its own bulk copies in flight, used while unwinding.
__device__ __forceinline__ void settle(uint32_t bar, uint32_t parity) {
  for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(bar, parity) && globaltimer_ns() - t0 < 200000000ull;) {
  }
}

// ------------------------------------------------------------------ producers
// Weight items in consumption order, for every unit and layer of this CTA (warp 0, one thread).
template <int D>
__device__ void weight_producer(const StackParams& p, uint32_t ring, const Bars& b, volatile int* abort_flag) {
  using C = Cfg<D>;
  int stage = 0;
  uint32_t phase = 0, pending = 0, pend_par = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x)
    for (int l = 0; l < p.n_layer && ok; ++l)
      for (int j = 0; j < C::kItems && ok; ++j) {
        if (!(ok = mbar_wait(b.empty(stage), phase ^ 1, abort_flag))) break;
        const uint32_t bytes = C::item_bytes(j);
        mbar_arrive_expect_tx(b.full(stage), bytes);
        bulk_g2s(ring + stage * C::kItemBytes, p.wimg + ((size_t)l * C::kItems + j) * C::kItemBytes, bytes,
                 b.full(stage));
        pending |= 1u << stage;
        pend_par = (pend_par & ~(1u << stage)) | (phase << stage);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1;
        }
      }
  if (!ok)
    for (int s = 0; s < p.stages; ++s)
      if ((pending >> s) & 1u) settle(b.full(s), (pend_par >> s) & 1u);
}

// The unit's K/V images of each layer (score mode; warp 3, one thread).  A layer's images are
// loaded once every slot that used the images now in shared memory has finished its
// attention on them: slot 1 releases them only in units where it holds a tile, and the unit
// before a single-tile unit may still have slot 1 at work on its last layer.
template <int D>
__device__ void kv_producer(const StackParams& p, uint32_t sKV, const Bars& b, volatile int* abort_flag) {
  uint32_t ph0 = 0, ph1 = 0;
  bool ok = true, pending = false, slot1_reads = false;
  uint32_t pend_par = 0, kv_phase = 0;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const Tile t0 = tile_of<D>(p, u, 0), t1 = tile_of<D>(p, u, 1);
    const uint32_t bytes = 2u * t0.Lp * D * 2u;
    for (int l = 0; l < p.n_layer && ok; ++l) {
      if (!(ok = mbar_wait(b.kv_empty(0), ph0 ^ 1, abort_flag))) break;
      ph0 ^= 1;
      if (slot1_reads) {   // slot 1's release of the previous images (its ph1-th release)
        if (!(ok = mbar_wait(b.kv_empty(1), ph1, abort_flag))) break;
        ph1 ^= 1;
      }
      slot1_reads = t1.active;
      if (bytes) {
        mbar_arrive_expect_tx(b.kv_full(), bytes);
        bulk_g2s(sKV, p.req[t0.r].kv + (size_t)l * bytes, bytes, b.kv_full());
        pending = true;
        pend_par = kv_phase;
      } else {
        mbar_arrive(b.kv_full());
      }
      kv_phase ^= 1;
    }
  }
  if (!ok && pending) settle(b.kv_full(), pend_par);
}

// ------------------------------------------------------------------ MMA issuer (one thread per slot)
template <int D, int SW, bool UM>
__device__ void mma_issuer(const StackParams& p, int slot, uint32_t tmem, uint32_t sA, uint32_t sKV, uint32_t ring,
                           uint32_t sOnes, const Bars& b, volatile int* abort_flag) {
  using C = Cfg<D>;
  constexpr uint32_t ID16 = idesc_f16(kM, 16);
  const uint32_t tY = tmem + kSlotCols * slot, tW = tY + D;
  const uint32_t e2m = b.e2m(slot), m2e = b.m2e(slot);
  int stage = 0;
  uint32_t phase = 0, ph_e = 0, ph_kv = 0, ph_mm = 0;
  bool ok = true, store_pending = false;
  auto wait_e = [&]() {
    ok = ok && mbar_wait(e2m, ph_e, abort_flag);
    ph_e ^= 1;
    tc_fence_after();
    return ok;
  };
  auto advance = [&]() {
    if (++stage == p.stages) {
      stage = 0;
      phase ^= 1;
    }
  };
  // D[dcol..] (+)= A x B^T (+ bias) for weight piece pi; A in shared memory (a = operand
  // base) or, for the FFN's second product, in tensor memory (a = column)
  auto piece = [&](int pi, uint32_t dcol, bool acc, bool a_tmem, uint32_t a) {
    const Piece pc = C::piece(pi);
    const bool first = pi == 0 || C::piece(pi - 1).item != pc.item;
    const bool last = pi == C::kPieces - 1 || C::piece(pi + 1).item != pc.item;
    if (!ok) return;
    if (first) {
      if (!(ok = mbar_wait(b.full(stage), phase, abort_flag))) return;
      tc_fence_after();
    }
    const uint32_t item = ring + stage * C::kItemBytes;
    const uint32_t id = idesc_f16(kM, pc.N);
#pragma unroll 1
    for (int kk = 0; kk < pc.K / 16; ++kk) {
      const uint64_t bd = sdesc(item + pc.off + kk * pc.N * 32, pc.N * 16, 128);
      const uint32_t accf = (kk > 0 || acc) ? 1u : 0u;
      if (a_tmem)   // the epilogue parts' fp16 hidden units: [0, 64), or [0, 32) and [64, 96)
        mma_bf16_ta(dcol, a + (Par<D>::P == 2 ? (kk & 3) * 8 + (kk >> 2) * 64 : kk * 8), bd, id, accf);
      else
        mma_bf16(dcol, sdesc(a + kk * 4096, 2048, 128), bd, id, accf);
    }
    if (pc.bias >= 0) mma_bf16(dcol, sdesc(sOnes, 2048, 128), sdesc(item + pc.bias, pc.N * 16, 128), id, 1u);
    if (last) {
      mma_commit(b.empty(stage));
      advance();
    }
  };
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const Tile t = tile_of<D>(p, u, slot);
    if (!t.active) {
      // the other slot works alone on this unit: release its weight items as they arrive
      for (int l = 0; l < p.n_layer && ok; ++l) {
        for (int j = 0; j < C::kItems && ok; ++j) {
          if (!(ok = mbar_wait(b.full(stage), phase, abort_flag))) break;
          mbar_arrive(b.empty(stage));
          advance();
        }
        ph_kv ^= 1;
      }
      continue;
    }
    const uint32_t idS = idesc_f16(kM, t.Lp > 0 ? t.Lp : 16);
    const uint32_t vimg = sKV + (uint32_t)t.Lp * D * 2;
    for (int l = 0; l < p.n_layer && ok; ++l) {
      // opaque per layer: keeps descriptor arithmetic from being hoisted into registers
      asm volatile("" : "+r"(sA), "+r"(sKV), "+r"(ring), "+r"(sOnes));
      if (!wait_e()) break;                            // A = LN1(y)
      piece(P_K, tW, false, false, sA);
      if (UM && store_pending) {                       // the last layer's images have left shared memory
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        store_pending = false;
      }
      mma_commit(m2e);
      if (!wait_e()) break;                            // own K read (user mode: K image written)
      piece(P_V, tW, false, false, sA);
      mma_commit(m2e);
      if (!wait_e()) break;                            // own V read (user mode: V image written)
      piece(P_Q, tW, false, false, sA);
      mma_commit(m2e);
      if (!wait_e()) break;                            // A = Q (score mode without users: attention output)
      if constexpr (UM) {
        const uint32_t bytes = 2u * t.Lp * D * 2u;
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                         p.req[t.r].kv + (size_t)l * bytes),
                     "r"(sKV), "r"(bytes)
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        store_pending = true;
      } else {
        ok = ok && mbar_wait(b.kv_full(), ph_kv, abort_flag);
        ph_kv ^= 1;
        tc_fence_after();
      }
      constexpr int HG = Groups<D, SW>::HG, HW = Groups<D, SW>::HW;
      const int ng = t.Lp > 0 ? Groups<D, SW>::NG : 0;
      for (int g = 0; g < ng && ok; ++g) {
        for (int i = 0; i < HG; ++i) {                 // scores of the group's heads
          const int h = g * HG + i;
          mma_bf16(tW + i * HW, sdesc(sA + h * 4096, 2048, 128),
                   sdesc(sKV + 2 * h * (t.Lp / 8) * 128, (t.Lp / 8) * 128, 128), idS, 0u);
        }
        mma_commit(m2e);
        if (!wait_e()) break;                          // numerators written
        for (int i = 0; i < HG; ++i) {                 // P V and the row sum beside them
          const int h = g * HG + i;
          const uint32_t pc = tW + i * HW;
          for (int kk = 0; kk < t.Lp / 16; ++kk) {
            mma_bf16_ta(pc + HW / 2, pc + kk * 8, sdesc(vimg + (2 * kk * (D / 8) + 2 * h) * 128, (D / 8) * 128, 128),
                        ID16, kk > 0 ? 1u : 0u);
            if (Par<D>::P == 1)   // with two epilogue parts the softmax adds the row sum itself
              mma_bf16_ta(pc + HW / 2 + 16, pc + kk * 8, sdesc(sOnes + kOnesBOff, 256, 128), ID16, kk > 0 ? 1u : 0u);
          }
        }
        if (!UM && g == ng - 1) mma_commit(b.kv_empty(slot));
        mma_commit(m2e);
        if (!wait_e()) break;                          // attention output of the group in A
      }
      if (!ok) break;
      if (!UM && ng == 0) mbar_arrive(b.kv_empty(slot));   // no product read the images
      piece(P_O, tY, true, false, sA);                // Y += attn Wo + bo
      mma_commit(m2e);
      if (!wait_e()) break;                            // A = LN2(y)
      piece(P_W1A, tW, false, false, sA);              // hidden (first half) + b1
      mma_commit(m2e);
      if (!wait_e()) break;                            // ReLU as fp16 in W[0, 64)
      piece(P_W2A, tY, true, true, tW);                // Y += relu W2 (first half of K)
      if constexpr (C::kFfnHalves == 2) {
        // the second half of the hidden units overwrites W: the first W2 product must be done
        mma_commit(b.mm(slot));
        ok = ok && mbar_wait(b.mm(slot), ph_mm, abort_flag);
        ph_mm ^= 1;
        tc_fence_after();
        piece(P_W1B, tW, false, false, sA);
        mma_commit(m2e);
        if (!wait_e()) break;
        piece(P_W2B, tY, true, true, tW);              // + b2
      }
      mma_commit(m2e);
    }
  }
  if (UM && store_pending) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  // drain every MMA still in flight before the tensor memory is released
  mma_commit(b.drain(slot));
  for (uint64_t t0 = globaltimer_ns(); !mbar_try_wait(b.drain(slot), 0) && globaltimer_ns() - t0 < 500000000ull;) {
  }
}

// ------------------------------------------------------------------ epilogue (two threads per row)
// The epilogue threads of a slot are P warps per TMEM lane quadrant: the thread of part p
// owns row m's columns [p D/P, (p + 1) D/P) in every row-wise phase (Y, LayerNorm, ReLU) and
// the heads h with h mod P = p in the attention; with two parts a row's LayerNorm statistics
// and its score are merged across them through shared memory.
struct Epi {
  uint32_t tY, tW;            // TMEM address of this row: residual, work area
  uint32_t sA, rowoff, sKV;
  int m, part;
  uint32_t e2m, m2e, ph;
  uint32_t gate, gph;         // the start gate of slot 1 in a unit of two tiles
  uint32_t xbar, xph, xbuf, xsel;   // the exchange with the row's other part
  int slot;
  bool paired;                 // both slots of the unit hold a tile
  const float* vec;
  volatile int* abort_flag;
  bool ok;
  // Slot 1 starts a unit of two tiles once slot 0 is well into it (through the attention of
  // its second head group, or through its own-V phase when the weight ring is two items
  // deep), so that the two slots' phases interleave: one slot's softmax runs while the
  // tensor core serves the other slot's projections.
  // (A warp takes every wait's outcome together, so that its lanes leave together when a
  // wait gives up and the single-lane arrivals below always see the whole warp.)
  __device__ __forceinline__ bool acquire() {
    if (paired && slot == 1) {
      ok = __all_sync(0xffffffffu, ok && mbar_wait(gate, gph, abort_flag));
      gph ^= 1;
    }
    return ok;
  }
  __device__ __forceinline__ void open_gate() {
    __syncwarp();
    if (paired && slot == 0 && (m & 31) == 0) mbar_arrive(gate);
  }
  // (the wait suspends between polls, leaving the issue slots to the other slot's warps)
  __device__ __forceinline__ bool wait() {
    ok = __all_sync(0xffffffffu, ok && mbar_wait_idle(m2e, ph, abort_flag));
    ph ^= 1;
    tc_fence_after();
    return ok;
  }
  // Each thread completes its tensor-memory stores and orders its shared-memory stores
  // before the tensor core's reads; then one lane per warp arrives for the whole warp.
  __device__ __forceinline__ void signal() {
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if ((m & 31) == 0) mbar_arrive(e2m);
  }
  // Two floats to the row's other part and its two back (the two buffers alternate, so a
  // buffer is rewritten only after the partner has passed the exchange that read it).
  __device__ __forceinline__ float2 xchg(float2 mine) {
    const uint32_t x = xbuf + xsel * (kMaxParts * kM * 8);
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(x + (part * kM + m) * 8), "f"(mine.x), "f"(mine.y)
                 : "memory");
    __syncwarp();
    if ((m & 31) == 0) mbar_arrive(xbar);
    ok = __all_sync(0xffffffffu, ok && mbar_wait(xbar, xph, abort_flag));
    xph ^= 1;
    float2 o;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(o.x), "=f"(o.y) : "r"(x + ((1 - part) * kM + m) * 8)
                 : "memory");
    xsel ^= 1;
    return o;
  }
};

// Packed fp32 pairs (one instruction for two lanes' worth of values).
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ float lo32(uint64_t r) { return __uint_as_float((uint32_t)r); }
__device__ __forceinline__ float hi32(uint64_t r) { return __uint_as_float((uint32_t)(r >> 32)); }

// s_lo += lo(a) lo(b), s_hi += hi(a) hi(b) for two fp16 pairs: the products are exact in
// fp32, the sums fp32.
__device__ __forceinline__ void fma_h2(float& s_lo, float& s_hi, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %2;\n\tmov.b32 {b0, b1}, %3;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\tfma.rn.f32.f16 %1, a1, b1, %1;\n\t}"
      : "+f"(s_lo), "+f"(s_hi)
      : "r"(a), "r"(b));
}

// This part's N columns of the row from tensor memory.
template <int N>
__device__ __forceinline__ void load_part(uint32_t taddr, float* y) {
#pragma unroll
  for (int c = 0; c < N / 16; ++c) tmem_ld16(taddr + 16 * c, y + 16 * c);
  tmem_wait_ld();
  reg_fence<N>(y);
}

// Row mean and 1/sqrt(var + eps) over D columns, of which this part holds y[0 .. D/P): each
// part's mean and sum of squared deviations (on packed pairs), merged with the other part's
// (Chan's update) when there are two.
template <int D>
__device__ __forceinline__ float2 row_stats(Epi& e, const float* y) {
  constexpr int P = Par<D>::P, N = D / P;
  uint64_t a[2] = {0ull, 0ull};
#pragma unroll
  for (int i = 0; i < N / 2; ++i) a[i & 1] = add_f32x2(a[i & 1], f32x2(y[2 * i], y[2 * i + 1]));
  const float mean = ((lo32(a[0]) + lo32(a[1])) + (hi32(a[0]) + hi32(a[1]))) * (1.f / N);
  const uint64_t nm = f32x2(-mean, -mean);
  a[0] = a[1] = 0ull;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const uint64_t d = add_f32x2(f32x2(y[2 * i], y[2 * i + 1]), nm);
    a[i & 1] = fma2(d, d, a[i & 1]);
  }
  const float m2 = (lo32(a[0]) + lo32(a[1])) + (hi32(a[0]) + hi32(a[1]));
  if constexpr (P == 1) {
    return make_float2(mean, rsqrtf(m2 * (1.f / D) + kLnEps));
  } else {
    const float2 o = e.xchg(make_float2(mean, m2));
    // the parts in a fixed order, so that both compute the same bits
    const float ma = e.part == 0 ? mean : o.x, mb = e.part == 0 ? o.x : mean;
    const float qa = e.part == 0 ? m2 : o.y, qb = e.part == 0 ? o.y : m2;
    const float dm = ma - mb;
    const float mu = 0.5f * (ma + mb);
    const float var = ((qa + qb) + dm * dm * (0.25f * D)) * (1.f / D);
    return make_float2(mu, rsqrtf(var + kLnEps));
  }
}

// The row standardized (LayerNorm without its gain and shift, which the next product's
// weights carry) -> this part's columns of the fp16 A operand row.
template <int D>
__device__ __forceinline__ void ln_to_A(Epi& e, const float* y) {
  constexpr int P = Par<D>::P;
  const float2 st = row_stats<D>(e, y);
  const uint64_t r2 = f32x2(st.y, st.y), n2 = f32x2(-st.x * st.y, -st.x * st.y);
#pragma unroll
  for (int kc = 0; kc < D / (8 * P); ++kc) {
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t v = fma2(f32x2(y[8 * kc + 2 * i], y[8 * kc + 2 * i + 1]), r2, n2);
      h[i] = pack_h2(lo32(v), hi32(v));
    }
    st_shared_v4(e.sA + (e.part * (D / (8 * P)) + kc) * 2048 + e.rowoff, h[0], h[1], h[2], h[3]);
  }
}

// This part's N hidden units of the work area -> fp16 -> ReLU (max with 0 on the pairs;
// rounding keeps the sign, so this equals rounding after the ReLU) -> the first N/2 columns
// of the same N (in place: every value is read before the first store).
template <int N>
__device__ __forceinline__ void relu_in_place(uint32_t tw) {
  float h[N];
#pragma unroll
  for (int c = 0; c < N / 32; ++c) tmem_ld32(tw + 32 * c, h + 32 * c);
  tmem_wait_ld();
  reg_fence<N>(h);
#pragma unroll
  for (int c = 0; c < N / 32; ++c) {
    uint32_t r[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t v = pack_h2(h[32 * c + 2 * i], h[32 * c + 2 * i + 1]);
      asm("max.f16x2 %0, %1, %2;" : "=r"(r[i]) : "r"(v), "r"(0u));
    }
    tmem_st16u(tw + 16 * c, r);
  }
}

// Softmax numerators of one head's row over its Lp key columns at `base` (keys >= L_u
// masked), with the own key's score `sself` (-inf when there is none) in the maximum: the
// numerators go back as fp16 pairs over the first Lp / 2 columns; returns the own key's
// numerator.  The row sum of the numerators comes from the tensor core (a product with a
// tile of ones, beside P V), so it adds exactly the fp16 values that P V weighs.
template <int SW, bool LEAN>
__device__ __forceinline__ float softmax_head(uint32_t base, int Lp, int L_u, float sself, float* rowsum = nullptr) {
  const int nb = Lp / 16;
  float mx;
  if constexpr (SW <= 64 && !LEAN) {
    float sv[SW];
#pragma unroll
    for (int c = 0; c < SW / 16; ++c)
      if (c < nb) tmem_ld16(base + 16 * c, sv + 16 * c);
    tmem_wait_ld();
    reg_fence<SW>(sv);
    if (L_u < SW) {   // keys past L_u (and unloaded chunks) out of the maximum
#pragma unroll
      for (int i = 0; i < SW; ++i)
        if (i >= L_u) sv[i] = -INFINITY;
    }
    float m4[4] = {sself, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int i = 0; i < SW; i += 8) {
      m4[0] = max3(m4[0], sv[i], sv[i + 1]);
      m4[1] = max3(m4[1], sv[i + 2], sv[i + 3]);
      m4[2] = max3(m4[2], sv[i + 4], sv[i + 5]);
      m4[3] = max3(m4[3], sv[i + 6], sv[i + 7]);
    }
    mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    const uint64_t l2 = f32x2(kL2E, kL2E), n2 = f32x2(-mx * kL2E, -mx * kL2E);
#pragma unroll
    for (int c = 0; c < SW / 16; ++c)
      if (c < nb) {
        uint32_t r[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint64_t x = fma2(f32x2(sv[16 * c + 2 * i], sv[16 * c + 2 * i + 1]), l2, n2);
          r[i] = exp2_h2(lo32(x), hi32(x));
        }
        tmem_st8u(base + 8 * c, r);
      }
  } else {
    // two passes over 16-key chunks: the maximum, then the numerators (chunk c's numerators
    // land in columns 8c .. 8c + 7, which only chunks up to c have occupied)
    mx = sself;
#pragma unroll 1
    for (int c = 0; c < nb; ++c) {
      float v[16];
      tmem_ld16(base + 16 * c, v);
      tmem_wait_ld();
      reg_fence<16>(v);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (16 * c + i < L_u) mx = fmaxf(mx, v[i]);
    }
    const uint64_t l2 = f32x2(kL2E, kL2E), n2 = f32x2(-mx * kL2E, -mx * kL2E);
    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int c = 0; c < nb; ++c) {
      float v[16];
      tmem_ld16(base + 16 * c, v);
      tmem_wait_ld();
      reg_fence<16>(v);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (16 * c + i >= L_u) v[i] = -INFINITY;
      uint32_t r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint64_t x = fma2(f32x2(v[2 * i], v[2 * i + 1]), l2, n2);
        r[i] = exp2_h2(lo32(x), hi32(x));
        if constexpr (LEAN) acc_h2(s4[(2 * i) & 3], s4[(2 * i + 1) & 3], r[i]);
      }
      tmem_st8u(base + 8 * c, r);
    }
    // LEAN: the numerators' row sum here (fp16 values added in fp32) instead of from the
    // tensor core
    if constexpr (LEAN) *rowsum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
  }
  return ex2(fmaf(sself, kL2E, -mx * kL2E));
}

// The two heads of a group (SW <= 64, two 64-column head regions from `base`), both in one
// thread: head 1's scores are read chunk by chunk into the registers that head 0's
// numerators have just left, so that their tensor-memory latency hides behind head 0's
// exponentials.
template <int SW>
__device__ __forceinline__ void softmax_two(uint32_t base, int Lp, int L_u, float ss0, float ss1, float* ps) {
  const int nb = Lp / 16;
  float sv[SW];
#pragma unroll
  for (int c = 0; c < SW / 16; ++c)
    if (c < nb) tmem_ld16(base + 16 * c, sv + 16 * c);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t hb = base + 64 * i;
    const float sself = i == 0 ? ss0 : ss1;
    tmem_wait_ld();
    reg_fence<SW>(sv);
    if (L_u < SW) {
#pragma unroll
      for (int k = 0; k < SW; ++k)
        if (k >= L_u) sv[k] = -INFINITY;
    }
    float m4[4] = {sself, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < SW; k += 8) {
      m4[0] = max3(m4[0], sv[k], sv[k + 1]);
      m4[1] = max3(m4[1], sv[k + 2], sv[k + 3]);
      m4[2] = max3(m4[2], sv[k + 4], sv[k + 5]);
      m4[3] = max3(m4[3], sv[k + 6], sv[k + 7]);
    }
    const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    const uint64_t l2 = f32x2(kL2E, kL2E), n2 = f32x2(-mx * kL2E, -mx * kL2E);
#pragma unroll
    for (int c = 0; c < SW / 16; ++c)
      if (c < nb) {
        uint32_t r[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t x = fma2(f32x2(sv[16 * c + 2 * k], sv[16 * c + 2 * k + 1]), l2, n2);
          r[k] = exp2_h2(lo32(x), hi32(x));
        }
        tmem_st8u(hb + 8 * c, r);
        if (i == 0) tmem_ld16(base + 64 + 16 * c, sv + 16 * c);
      }
    ps[i] = ex2(fmaf(sself, kL2E, -mx * kL2E));
  }
}

// Attention output of head h (own index k) from its P V product and row sum at `hb`:
// o = (ps v_own + P V) / (sum + ps) -> the head's 16 columns of A.
template <int D, bool UM>
__device__ __forceinline__ void finish_head(const Epi& e, uint32_t hb, int hw, int h, int k, float ps,
                                            const uint32_t* vreg, float rowsum) {
  constexpr int NP = Cfg<D>::kNH / Par<D>::P;
  float o[16];
  tmem_ld16(hb + hw / 2, o);
  float sum = rowsum;
  if constexpr (Par<D>::P == 1) sum = tmem_ld1(hb + hw / 2 + 16);
  tmem_wait_ld();
  reg_fence<16>(o);
  asm volatile("" : "+f"(sum));
  const float li = rcp_approx(sum + ps);
  if constexpr (UM) {
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j] *= li;
  } else {
    uint32_t vv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      vv[j] = vreg[j];
#pragma unroll
      for (int kk = 1; kk < NP; ++kk) vv[j] = k == kk ? vreg[8 * kk + j] : vv[j];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      o[2 * j] = fmaf(ps, h_lo(vv[j]), o[2 * j]) * li;
      o[2 * j + 1] = fmaf(ps, h_hi(vv[j]), o[2 * j + 1]) * li;
    }
  }
  st_row8h(e.sA + (2 * h) * 2048 + e.rowoff, o);
  st_row8h(e.sA + (2 * h + 1) * 2048 + e.rowoff, o + 8);
}

template <int D, int SW, bool UM, bool OG>
__device__ __forceinline__ void epi_tile(const StackParams& p, const Tile& t, Epi& e) {
  constexpr int P = Par<D>::P;
  constexpr int NH = Cfg<D>::kNH;
  constexpr int NP = NH / P;                   // heads of this part: P k + part
  constexpr int DP = D / P;                    // columns of this part
  const int m = e.m, part = e.part;
  const bool live = m < t.rows;
  if (!e.acquire()) return;
  // ---- Y = token + s_d, this part's columns (rows past the tile's end are zero, never stored)
  {
    float y[DP];
    const float4* sd4 = reinterpret_cast<const float4*>(p.domain_emb + (size_t)t.dom * D + part * DP);
    if constexpr (OG) {   // bf16 tokens, widened exactly
      const uint4* src = reinterpret_cast<const uint4*>(p.tokens_h + (size_t)(t.row0 + m) * D + part * DP);
#pragma unroll
      for (int c = 0; c < DP / 8; ++c) {
        const uint4 u = live ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const float4 d0 = __ldg(sd4 + 2 * c), d1 = __ldg(sd4 + 2 * c + 1);
        const float d[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          y[8 * c + 2 * i] = live ? __uint_as_float(w[i] << 16) + d[2 * i] : 0.f;
          y[8 * c + 2 * i + 1] = live ? __uint_as_float(w[i] & 0xFFFF0000u) + d[2 * i + 1] : 0.f;
        }
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(
          (UM ? p.req[t.r].utokens + (size_t)m * D : p.tokens + (size_t)(t.row0 + m) * D) + part * DP);
#pragma unroll
      for (int c = 0; c < DP / 4; ++c) {
        const float4 u = live ? __ldg(src + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 d = __ldg(sd4 + c);
        y[4 * c] = live ? u.x + d.x : 0.f;
        y[4 * c + 1] = live ? u.y + d.y : 0.f;
        y[4 * c + 2] = live ? u.z + d.z : 0.f;
        y[4 * c + 3] = live ? u.w + d.w : 0.f;
      }
    }
#pragma unroll
    for (int c = 0; c < DP / 16; ++c) tmem_st16(e.tY + part * DP + 16 * c, y + 16 * c);
    tmem_wait_st();
  }
  // (Y is re-read from tensor memory at the top of every layer, so that no register copy of
  // it stays live through the layer)
  for (int l = 0; l < p.n_layer; ++l) {
    if (l > 0 && !e.wait()) return;   // the previous layer's FFN product is in Y
    {
      float y[DP];
      load_part<DP>(e.tY + part * DP, y);
      ln_to_A<D>(e, y);
    }
    e.signal();
    // ---- own K and V of this part's heads (user mode: their columns of this row of the
    // layer's K and V^T images), two heads at a time
    uint32_t kreg[UM ? 1 : 8 * NP], vreg[UM ? 1 : 8 * NP];
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      if (!e.wait()) return;
#pragma unroll
      for (int k2 = 0; k2 < NP; k2 += 2) {
        float x[32];
#pragma unroll
        for (int j = 0; j < 2; ++j) tmem_ld16(e.tW + 16 * (P * (k2 + j) + part), x + 16 * j);
        tmem_wait_ld();
        reg_fence<32>(x);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int k = k2 + j, h = P * k + part;
          if constexpr (UM) {
            if (m < t.Lp) {
              const bool real = m < t.L_u;
              if (pass == 0) {   // K image [Lp x D]: row m, eight columns per core-matrix row
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                  float v[8];
#pragma unroll
                  for (int i = 0; i < 8; ++i) v[i] = real ? x[16 * j + 8 * c + i] : 0.f;
                  st_row8h(e.sKV + ((2 * h + c) * (t.Lp / 8) + (m >> 3)) * 128 + (m & 7) * 16, v);
                }
              } else {           // V^T image [D x Lp]: column m
                const uint32_t vb = e.sKV + t.Lp * D * 2 + (m >> 3) * (D / 8) * 128 + (m & 7) * 2;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const int d = 16 * h + i;
                  const __half hv = __float2half_rn(real ? x[16 * j + i] : 0.f);
                  asm volatile("st.shared.b16 [%0], %1;" ::"r"(vb + (d >> 3) * 128 + (d & 7) * 16),
                               "h"(*reinterpret_cast<const unsigned short*>(&hv))
                               : "memory");
                }
              }
            }
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              if (pass == 0)
                kreg[8 * k + i] = pack_h2(x[16 * j + 2 * i], x[16 * j + 2 * i + 1]);
              else
                vreg[8 * k + i] = pack_h2(x[16 * j + 2 * i], x[16 * j + 2 * i + 1]);
            }
          }
        }
      }
      e.signal();
      if (l == 0 && pass == 1 && p.gate_phase == 0) e.open_gate();
    }
    // ---- Q of this part's heads (pre-scaled by 1/sqrt(d_h) through its weights) -> A; own
    // score per head
    float sself[NP];
    float rsc[OG ? NP : 1];   // OG: the own tokens' numerator sum relative to their maximum
    if (!e.wait()) return;
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const int h = P * k + part;
      float q[16];
      tmem_ld16(e.tW + 16 * h, q);
      tmem_wait_ld();
      reg_fence<16>(q);
      uint32_t qp[8];   // the head's query as the fp16 pairs the score product reads
#pragma unroll
      for (int i = 0; i < 8; ++i) qp[i] = pack_h2(q[2 * i], q[2 * i + 1]);
      if constexpr (UM) {
        sself[k] = -INFINITY;
      } else if constexpr (OG) {
        // the own candidate's lt tokens sit in lanes g0 .. g0 + lt - 1: their keys and values
        // come by shuffle; an online softmax over them leaves their largest score (which
        // joins the user keys' maximum), the sum R of their numerators relative to it, and
        // their numerator-weighted mean value, which replaces the own value: the attention
        // output is then (ps R vmean + P V) / (sum + ps R), ps the numerator of the largest
        const int g0 = (m & 31) & ~(p.lt - 1);
        float mo = -INFINITY, R = 0.f, va[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) va[i] = 0.f;
#pragma unroll 1
        for (int j = 0; j < p.lt; ++j) {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) fma_h2(s0, s1, qp[i], __shfl_sync(0xffffffffu, kreg[8 * k + i], g0 + j));
          const float sj = s0 + s1;
          if (sj > mo) {
            const float c = ex2((mo - sj) * kL2E);
            R *= c;
#pragma unroll
            for (int i = 0; i < 16; ++i) va[i] *= c;
            mo = sj;
          }
          const float rj = ex2((sj - mo) * kL2E);
          R += rj;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t vv = __shfl_sync(0xffffffffu, vreg[8 * k + i], g0 + j);
            va[2 * i] = fmaf(rj, h_lo(vv), va[2 * i]);
            va[2 * i + 1] = fmaf(rj, h_hi(vv), va[2 * i + 1]);
          }
        }
        sself[k] = mo;
        rsc[k] = R;
        const float ri = 1.f / R;
#pragma unroll
        for (int i = 0; i < 8; ++i) vreg[8 * k + i] = pack_h2(va[2 * i] * ri, va[2 * i + 1] * ri);
      } else {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) fma_h2(s0, s1, qp[i], kreg[8 * k + i]);
        sself[k] = s0 + s1;
      }
      if (UM || t.Lp > 0) {
        st_shared_v4(e.sA + (2 * h) * 2048 + e.rowoff, qp[0], qp[1], qp[2], qp[3]);
        st_shared_v4(e.sA + (2 * h + 1) * 2048 + e.rowoff, qp[4], qp[5], qp[6], qp[7]);
      } else {             // no user keys: the attention output is the own value
        if constexpr (!UM) {
          st_shared_v4(e.sA + (2 * h) * 2048 + e.rowoff, vreg[8 * k], vreg[8 * k + 1], vreg[8 * k + 2],
                       vreg[8 * k + 3]);
          st_shared_v4(e.sA + (2 * h + 1) * 2048 + e.rowoff, vreg[8 * k + 4], vreg[8 * k + 5], vreg[8 * k + 6],
                       vreg[8 * k + 7]);
        }
      }
    }
    e.signal();
    if (l == 0 && t.Lp == 0 && p.gate_phase == 1) e.open_gate();
    // ---- attention, one head group at a time.  Two heads per group: with two parts each
    // takes one (head 2g + part), with one part the thread takes both; one head per group:
    // the head's own part does it and the other waits.
    constexpr int HG = Groups<D, SW>::HG, HW = Groups<D, SW>::HW;
    if (t.Lp > 0) {
#pragma unroll 1
      for (int g = 0; g < Groups<D, SW>::NG; ++g) {
        if (!e.wait()) return;   // scores of group g
        if constexpr (HG == 2 && P == 1) {
          float ps[2];
          float s0 = sself[0], s1 = sself[1];
#pragma unroll
          for (int k = 2; k < NP; k += 2) {
            s0 = 2 * g == k ? sself[k] : s0;
            s1 = 2 * g == k ? sself[k + 1] : s1;
          }
          softmax_two<SW>(e.tW, t.Lp, t.L_u, s0, s1, ps);
          if constexpr (OG) {
#pragma unroll
            for (int k = 0; k < NP; k += 2) {
              ps[0] = 2 * g == k ? ps[0] * rsc[k] : ps[0];
              ps[1] = 2 * g == k ? ps[1] * rsc[k + 1] : ps[1];
            }
          }
          e.signal();
          if (!e.wait()) return;   // P V and the row sums of group g
#pragma unroll
          for (int i = 0; i < 2; ++i)
            finish_head<D, UM>(e, e.tW + i * HW, HW, 2 * g + i, 2 * g + i, ps[i], vreg, 0.f);
        } else {
          const int h = HG == 2 ? 2 * g + part : g;
          const bool mine = h % P == part;
          const int k = h / P;                       // own index of head h
          const uint32_t hb = e.tW + (HG == 2 ? part : 0) * HW;
          float ss = sself[0];
#pragma unroll
          for (int j = 1; j < NP; ++j) ss = k == j ? sself[j] : ss;
          float ps = 0.f, rowsum = 0.f;
          if (mine) ps = softmax_head<SW, P == 2>(hb, t.Lp, t.L_u, ss, &rowsum);
          if constexpr (OG) {
            float rs = rsc[0];
#pragma unroll
            for (int j = 1; j < NP; ++j) rs = k == j ? rsc[j] : rs;
            ps *= rs;
          }
          e.signal();
          if (!e.wait()) return;   // P V and the row sums of group g
          if (mine) finish_head<D, UM>(e, hb, HW, h, k, ps, vreg, rowsum);
        }
        e.signal();
        if (l == 0 && g == (Groups<D, SW>::NG > 1 ? 1 : 0) && p.gate_phase == 1) e.open_gate();
      }
    }
    // ---- LN2 -> A
    if (!e.wait()) return;        // Y += attn Wo + bo
    {
      float y[DP];
      load_part<DP>(e.tY + part * DP, y);
      ln_to_A<D>(e, y);
    }
    e.signal();
    // ---- ReLU(hidden) -> fp16 A operand in the work area, a 128-unit half at a time
#pragma unroll
    for (int half = 0; half < Cfg<D>::kFfnHalves; ++half) {
      if (!e.wait()) return;
      relu_in_place<128 / P>(e.tW + (128 / P) * part);
      e.signal();
    }
  }
  // ---- head: w . LN_f(y) + b (w folded with the final LayerNorm's gain); with two parts
  // their halves of the dot product are added in a fixed order
  if (!e.wait()) return;
  if (UM) return;
  float y[DP];
  load_part<DP>(e.tY + part * DP, y);
  const float2 st = row_stats<D>(e, y);
  const float* vf = e.vec + part * DP;
  float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < DP / 8; ++c) {
    float w[8];
    ld8(vf + 8 * c, w);
#pragma unroll
    for (int i = 0; i < 8; ++i) a4[i & 3] = fmaf((y[8 * c + i] - st.x) * st.y, w[i], a4[i & 3]);
  }
  const float mine = (a4[0] + a4[1]) + (a4[2] + a4[3]);
  float dot = mine;
  if constexpr (P == 2) {
    const float other = e.xchg(make_float2(mine, 0.f)).x;
    dot = part == 0 ? mine + other : other + mine;
  }
  if constexpr (OG) {
    // the candidate's score: the mean of its lt tokens' scores, summed over its lanes in a
    // fixed butterfly order (lt is a power of two)
    float sc = dot + e.vec[D];
    for (int off = 1; off < p.lt; off <<= 1) sc += __shfl_xor_sync(0xffffffffu, sc, off);
    if (live && part == 0 && (m & (p.lt - 1)) == 0) p.scores[(t.row0 + m) / p.lt] = sc * (1.f / p.lt);
  } else {
    if (live && part == 0) p.scores[t.row0 + m] = dot + e.vec[D];
  }
}

template <int D, int SW, bool UM, bool OG>
__device__ void epilogue(const StackParams& p, int slot, uint32_t tmem, uint32_t sA, uint32_t sKV, uint32_t sOnes,
                         const float* vec, const Bars& b, uint32_t xbuf, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Epi e;
  const int q = warp & 3;
  e.m = q * 32 + lane;
  e.part = ((warp - 4) >> 2) % Par<D>::P;
  e.tY = tmem + ((uint32_t)(q * 32) << 16) + kSlotCols * slot;
  e.tW = e.tY + D;
  e.sA = sA;
  e.rowoff = (e.m >> 3) * 128 + (e.m & 7) * 16;
  e.sKV = sKV;
  e.e2m = b.e2m(slot);
  e.m2e = b.m2e(slot);
  e.ph = 0;
  e.gate = b.tok(0);
  e.gph = 0;
  e.xbar = b.xch(slot, q);
  e.xph = 0;
  e.xbuf = xbuf;
  e.xsel = 0;
  e.slot = slot;
  e.vec = vec;
  e.abort_flag = abort_flag;
  e.ok = true;
  for (int u = blockIdx.x; u < p.n_units && e.ok; u += gridDim.x) {
    const Tile t = tile_of<D>(p, u, slot);
    e.paired = p.pair && tile_of<D>(p, u, 1).active;
    if (t.active) epi_tile<D, SW, UM, OG>(p, t, e);
  }
}

// OG: candidates of p.lt tokens each (lt consecutive rows of a tile, adjacent lanes of one
// warp), every token attending to its own candidate's tokens as well as to the user.
template <int D, int SW, bool UM, bool OG>
__global__ void __launch_bounds__(Par<D>::kThreads, 1) stack_kernel(const __grid_constant__ StackParams p) {
  constexpr int kSlotThreads = Par<D>::kSlotThreads;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t sA0 = base, sKV = base + p.off_kv, ring = base + p.off_ring, sOnes = base + p.off_ones;
  const Bars b{base + p.off_bar};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + p.off_bar + 8 * kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + p.off_bar + 8 * kNumBars + 8);
  const float* vec = p.off_vec >= 0 ? reinterpret_cast<const float*>(smem + p.off_vec) : p.vec;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(b.full(s), 1);
      mbar_init(b.empty(s), p.pair ? 2 : 1);
    }
    mbar_init(b.kv_full(), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(b.kv_empty(s), 1);
      mbar_init(b.e2m(s), kSlotThreads / 32);
      mbar_init(b.m2e(s), 1);
      mbar_init(b.mm(s), 1);
      mbar_init(b.drain(s), 1);
      mbar_init(b.tok(s), kSlotThreads / 32);
    }
    for (int i = 0; i < 8; ++i) mbar_init(b.xch(i >> 2, i & 3), Par<D>::P);
    *abort_flag = 0;
    mbar_fence_init();
    // The grid's weight images (and, in score mode, one layer's K/V images of this CTA's
    // first unit) into L2 at once: otherwise every CTA misses on the same item at the same
    // time when the launch follows kernels that have cycled L2.
    prefetch_l2_share(p.wimg, (size_t)p.n_layer * Cfg<D>::kItems * Cfg<D>::kItemBytes);
    if (!UM && (int)blockIdx.x < p.n_units) {
      const Tile t0 = tile_of<D>(p, blockIdx.x, 0);
      const uint32_t kvb = 2u * t0.Lp * D * 2u;
      if (kvb) prefetch_l2(p.req[t0.r].kv + (size_t)(blockIdx.x % p.n_layer) * kvb, kvb);
    }
  }
  if (warp == 3) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // constant operands: the ones tile (columns 0 and 1 of every row are 1) and the vectors
  if (threadIdx.x >= 128) {
    const int t = threadIdx.x - 128;
    if (t < kM) {
      const float one2[8] = {1.f, 1.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, zero[8] = {};
      const uint32_t ro = (t >> 3) * 128 + (t & 7) * 16;
      st_row8h(sOnes + ro, one2);
      st_row8h(sOnes + 2048 + ro, zero);
      if (t < 32) st_shared_v4(sOnes + kOnesBOff + 16 * t, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
    }
    if (p.off_vec >= 0) {
      const int nvec = vec_floats<D>();
      float* sv = reinterpret_cast<float*>(smem + p.off_vec);
      for (int i = t; i < nvec; i += 2 * kSlotThreads) sv[i] = __ldg(p.vec + i);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(Par<D>::kCtlRegs));
    if (lane == 0) {
      if (warp == 0) weight_producer<D>(p, ring, b, abort_flag);
      if (warp == 1) mma_issuer<D, SW, UM>(p, 0, tmem, sA0, sKV, ring, sOnes, b, abort_flag);
      if (warp == 2 && p.pair) mma_issuer<D, SW, UM>(p, 1, tmem, sA0 + kM * D * 2, sKV, ring, sOnes, b, abort_flag);
      if (warp == 3 && !UM) kv_producer<D>(p, sKV, b, abort_flag);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(Par<D>::kEpiRegs));
    const int slot = (warp - 4) / (4 * Par<D>::P);
    if (slot == 0 || p.pair)
      epilogue<D, SW, UM, OG>(p, slot, tmem, sA0 + slot * kM * D * 2, sKV, sOnes, vec, b,
                          base + p.off_xch + slot * kXchBytes, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, STATUS_KERNEL_TIMEOUT);
}

// ------------------------------------------------------------------ host: operand images

uint16_t f16_bits(float f) {
  const __half h = __float2half_rn(f);
  uint16_t u;
  memcpy(&u, &h, 2);
  return u;
}
float f16_value(uint16_t u) {
  __half h;
  memcpy(&h, &u, 2);
  return __half2float(h);
}

// B operand [N x K] of the product x W (W [K_total][ld] row-major, columns n0.., rows k0..),
// scaled by `scale`, in the core-matrix layout, fp16.
void put_B(uint16_t* dst, const float* W, int ld, int n0, int k0, int N, int K, float scale) {
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      dst[((size_t)(k / 8) * (N / 8) + n / 8) * 64 + (n % 8) * 8 + (k % 8)] =
          f16_bits(W[(size_t)(k0 + k) * ld + n0 + n] * scale);
}
// Bias tile [N x 16]: column 0 the fp16 nearest to b[n0+n] * scale, column 1 the fp16 of the rest.
void put_bias(uint16_t* dst, const float* bias, int n0, int N, float scale) {
  for (int n = 0; n < N; ++n) {
    const float v = bias[n0 + n] * scale;
    const uint16_t hi = f16_bits(v);
    const uint16_t lo = f16_bits(v - f16_value(hi));
    for (int k = 0; k < 16; ++k)
      dst[((size_t)(k / 8) * (N / 8) + n / 8) * 64 + (n % 8) * 8 + (k % 8)] = k == 0 ? hi : k == 1 ? lo : 0;
  }
}

// W' = diag(g) W scale and b' = (beta W + b) scale for a product that follows a LayerNorm with
// gain g and shift beta (fp64 on the host; W [K][ld] row-major, columns n0 .. n0 + N - 1).
void fold_ln(const float* W, int ld, int n0, int K, int N, const float* g, const float* beta, const float* bias,
             float scale, std::vector<float>& Wf, std::vector<float>& bf) {
  Wf.assign((size_t)K * N, 0.f);
  bf.assign(N, 0.f);
  for (int n = 0; n < N; ++n) {
    double acc = bias[n0 + n];
    for (int k = 0; k < K; ++k) {
      const double w = W[(size_t)k * ld + n0 + n];
      Wf[(size_t)k * N + n] = (float)(w * g[k] * scale);
      acc += (double)beta[k] * w;
    }
    bf[n] = (float)(acc * scale);
  }
}

template <int D>
void build_layer_items(uint8_t* li, const tr_layer_weights& L) {
  using C = Cfg<D>;
  const int H = 2 * D;
  auto at = [&](int pi, int off) {
    const Piece pc = C::piece(pi);
    return reinterpret_cast<uint16_t*>(li + (size_t)pc.item * C::kItemBytes + off);
  };
  std::vector<float> Wf, bf;
  // K, V, Q follow LN1; Q's weights and bias also carry 1/sqrt(d_h) = 1/4
  const float* Wn[3] = {L.Wk, L.Wv, L.Wq};
  const float* bn[3] = {L.bk, L.bv, L.bq};
  const float sc[3] = {1.f, 1.f, 0.25f};
  for (int j = 0; j < 3; ++j) {
    const Piece pc = C::piece(j);
    fold_ln(Wn[j], D, 0, D, D, L.ln1_g, L.ln1_b, bn[j], sc[j], Wf, bf);
    put_B(at(j, pc.off), Wf.data(), D, 0, 0, D, D, 1.f);
    put_bias(at(j, pc.bias), bf.data(), 0, D, 1.f);
  }
  {
    const Piece pc = C::piece(P_O);
    put_B(at(P_O, pc.off), L.Wo, D, 0, 0, D, D, 1.f);
    put_bias(at(P_O, pc.bias), L.bo, 0, D, 1.f);
  }
  for (int hf = 0; hf < C::kFfnHalves; ++hf) {
    const int p1 = hf == 0 ? P_W1A : P_W1B, p2 = hf == 0 ? P_W2A : P_W2B;
    const Piece a = C::piece(p1), b = C::piece(p2);
    fold_ln(L.W1, H, 128 * hf, D, 128, L.ln2_g, L.ln2_b, L.b1, 1.f, Wf, bf);   // hidden units 128 hf ..
    put_B(at(p1, a.off), Wf.data(), 128, 0, 0, 128, D, 1.f);
    put_bias(at(p1, a.bias), bf.data(), 0, 128, 1.f);
    put_B(at(p2, b.off), L.W2, D, 0, 128 * hf, D, 128, 1.f);            // rows 128 hf .. of W2
    if (b.bias >= 0) put_bias(at(p2, b.bias), L.b2, 0, D, 1.f);
  }
}

// Whether every fp16 operand of the stack stays far inside fp16's range: the standardized
// rows are bounded by sqrt(D); a product's outputs by that bound times the largest column
// sum of |g o W| plus the largest |folded bias|; the attention output by the bound of V;
// ReLU by the bound of its input; the folded weights by max |g| max |W|.
bool fp16_operands_safe(const tr_model_desc& d, const tr_model_weights* w) {
  const int D = d.D, H = d.ffn_hidden;
  auto amax = [](const float* p, size_t n) {
    double m = 0;
    for (size_t i = 0; i < n; ++i) m = std::max(m, (double)fabsf(p[i]));
    return m;
  };
  // bound of z W' + b' with W' = diag(g) W, b' = beta W + b, |z_k| <= sqrt(D)
  auto out_bound = [&](const float* W, int K, int N, const float* g, const float* beta, const float* b) {
    double m = 0;
    for (int n = 0; n < N; ++n) {
      double s = 0, c = b ? fabs((double)b[n]) : 0.0;
      for (int k = 0; k < K; ++k) {
        s += fabs((double)W[(size_t)k * N + n] * g[k]);
        c += fabs((double)W[(size_t)k * N + n] * beta[k]);
      }
      m = std::max(m, s * sqrt((double)K) + c);
    }
    return m;
  };
  const double limit = 16384.0;
  for (int l = 0; l < d.n_layer; ++l) {
    const tr_layer_weights& L = w->layers[l];
    const double q = out_bound(L.Wq, D, D, L.ln1_g, L.ln1_b, L.bq);
    const double k = out_bound(L.Wk, D, D, L.ln1_g, L.ln1_b, L.bk);
    const double v = out_bound(L.Wv, D, D, L.ln1_g, L.ln1_b, L.bv);
    const double h = out_bound(L.W1, D, H, L.ln2_g, L.ln2_b, L.b1);
    if (!(q < limit && k < limit && v < limit && h < limit)) return false;
    const double gmax = std::max(amax(L.ln1_g, D), amax(L.ln2_g, D));
    const double wmax = std::max({amax(L.Wq, (size_t)D * D), amax(L.Wk, (size_t)D * D), amax(L.Wv, (size_t)D * D),
                                  amax(L.Wo, (size_t)D * D), amax(L.W1, (size_t)D * H), amax(L.W2, (size_t)H * D)});
    if (!(wmax * std::max(gmax, 1.0) < limit)) return false;
  }
  return true;
}

}  // namespace

bool tc_stack_supported(const tr_model* m) { return m->tc_stack != nullptr; }

tr_status tc_build_comp(tr_model* m, const tr_model_weights* w);

template <int D>
tr_status build_stack_images(tr_model* m, const tr_model_weights* w) {
  using C = Cfg<D>;
  const tr_model_desc& d = m->desc;
  const int N = d.n_layer;
  std::vector<uint8_t> img((size_t)N * C::kItems * C::kItemBytes, 0);
  std::vector<float> vec(vec_floats<D>(), 0.f);
  for (int l = 0; l < N; ++l) build_layer_items<D>(img.data() + (size_t)l * C::kItems * C::kItemBytes, w->layers[l]);
  float* vf = vec.data();
  double bh = w->b_head;
  for (int j = 0; j < D; ++j) {
    vf[j] = (float)((double)w->w_head[j] * w->lnf_g[j]);
    bh += (double)w->w_head[j] * w->lnf_b[j];
  }
  vf[D] = (float)bh;
  const size_t img_bytes = img.size(), vec_bytes = vec.size() * 4;
  const size_t total = img_bytes + ((vec_bytes + 255) & ~size_t(255));
  if (cudaMalloc(&m->tc_blob, total) != cudaSuccess) {
    cudaGetLastError();
    return fail(TR_ERR_NOMEM, "tensor-core weight images: allocation of %zu bytes failed", total);
  }
  m->tc_bytes = total;
  TR_CUDA_TRY(cudaMemcpy(m->tc_blob, img.data(), img_bytes, cudaMemcpyHostToDevice));
  TR_CUDA_TRY(cudaMemcpy((uint8_t*)m->tc_blob + img_bytes, vec.data(), vec_bytes, cudaMemcpyHostToDevice));
  m->tc_stack = m->tc_blob;
  m->tc_stack_layer_bytes = (size_t)C::kItems * C::kItemBytes;
  m->tc_vec = reinterpret_cast<const float*>((uint8_t*)m->tc_blob + img_bytes);
  m->tc_vec_layer_floats = 0;
  return TR_OK;
}

tr_status tc_build(tr_model* m, const tr_model_weights* w) {
  const tr_model_desc& d = m->desc;
  TR_TRY(tc_build_comp(m, w));
  if (!(d.dtype == TR_BF16 && (d.D == 64 || d.D == 128) && d.ffn_hidden == 2 * d.D && d.n_head * 16 == d.D))
    return TR_OK;
  if (!fp16_operands_safe(d, w)) return TR_OK;    // the CUDA-core path serves this model
  return d.D == 128 ? build_stack_images<128>(m, w) : build_stack_images<64>(m, w);
}

namespace {

// Shared-memory layout of one launch; false when it does not fit.
template <int D>
bool plan_smem(StackParams& p, int n_layer, int lp_max, bool pair, int& smem_bytes) {
  const int a_bytes = (pair ? 2 : 1) * kM * D * 2;
  p.off_kv = a_bytes;
  const int kv_bytes = 2 * lp_max * D * 2;
  p.off_ones = p.off_kv + ((kv_bytes + 1023) & ~1023);
  p.off_xch = p.off_ones + kOnesBytes;
  p.off_ring = p.off_xch + 2 * kXchBytes;
  const int vec_bytes = vec_floats<D>() * 4;
  const int fixed = p.off_ring + kBarArea;
  int stages = std::min(kMaxStages, (kSmemLimit - fixed - vec_bytes) / Cfg<D>::kItemBytes);
  bool vec_in_smem = true;
  if (stages < 2) {
    vec_in_smem = false;
    stages = std::min(kMaxStages, (kSmemLimit - fixed) / Cfg<D>::kItemBytes);
  }
  if (stages < 2) return false;
  p.stages = stages;
  // slot 0 runs items K, V (and Q) of the unit's first layer before slot 1 starts: it needs
  // a third stage to reach the attention alone (D = 64 keeps all four projections in one item)
  p.gate_phase = (D == 128 && stages < 3) ? 0 : 1;
  int off = p.off_ring + stages * Cfg<D>::kItemBytes;
  if (vec_in_smem) {
    p.off_vec = off;
    off += (vec_bytes + 15) & ~15;
  } else {
    p.off_vec = -1;
  }
  p.off_bar = off;
  smem_bytes = off + kBarArea;
  return smem_bytes <= kSmemLimit;
}

template <int D, int SW, bool UM, bool OG = false>
tr_status launch(int grid, const StackParams& p, int smem, cudaStream_t st) {
  auto k = stack_kernel<D, SW, UM, OG>;
  TR_TRY(ensure_smem_attr((const void*)k, kSmemLimit));
  k<<<grid, Par<D>::kThreads, smem, st>>>(p);
  TR_LAUNCH_CHECK(UM ? "stack_kernel (user side)" : "stack_kernel");
  return TR_OK;
}

// lt = 0: one fp32 token per candidate; lt >= 1: lt bf16 tokens per candidate (the tile
// rows are then tokens, lt to a candidate).
template <int D>
tr_status score_launch(const tr_model* m, const void* tokens, const int64_t* req_offsets, const void* const* kv,
                       const int32_t* L_u, const int32_t* domain, int R, float* scores, cudaStream_t st,
                       int lt = 0) {
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  StackParams p{};
  const bool og = lt > 0;
  const int rows_per = og ? lt : 1;
  if (og) {
    p.tokens_h = static_cast<const uint16_t*>(tokens);
    p.lt = lt;
  } else {
    p.tokens = static_cast<const float*>(tokens);
    p.lt = 1;
  }
  p.scores = scores;
  p.wimg = static_cast<const uint8_t*>(m->tc_stack);
  p.vec = m->tc_vec;
  p.domain_emb = m->domain_emb;
  p.status = ds->status;
  p.n_layer = m->desc.n_layer;
  p.pair = 1;
  int sms = 148, dev = 0;
  TR_CUDA_TRY(cudaGetDevice(&dev));
  TR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  // Units: pairs of consecutive tiles of one request (the request's last unit is a single
  // tile when its tile count is odd).  Units go to the CTAs round robin; when the last round
  // is partial, its pairs are split into single tiles (as many as there are idle CTAs in that
  // round), which spreads the round over more SMs.
  int k = 0, lp_max = 0;
  int tiles_of[TR_MAX_REQUESTS], pairs_of[TR_MAX_REQUESTS];
  int units = 0;
  for (int r = 0; r < R; ++r) {
    const int64_t nr = req_offsets[r + 1] - req_offsets[r];
    if (nr == 0) continue;
    p.req[k].kv = static_cast<const uint8_t*>(kv[r]);
    p.req[k].cand_off = req_offsets[r] * rows_per;
    p.req[k].n = nr * rows_per;
    p.req[k].L_u = L_u[r];
    p.req[k].domain = domain[r];
    lp_max = std::max(lp_max, round_up16(L_u[r]));
    tiles_of[k] = (int)((nr * rows_per + kM - 1) / kM);
    pairs_of[k] = tiles_of[k] / 2;
    units += tiles_of[k] - pairs_of[k];
    ++k;
  }
  if (units > 0) {
    const int rem = units % sms;                 // units of the partial last round (0: none)
    int window = rem, room = rem ? sms - rem : 0;
    for (int q = k - 1; q >= 0 && window > 0 && room > 0; --q) {
      const int singles = tiles_of[q] - 2 * pairs_of[q];
      int in_window = std::min(window, singles + pairs_of[q]);
      const int pairs_in_window = std::max(0, in_window - singles);
      const int split = std::min(pairs_in_window, room);
      pairs_of[q] -= split;
      room -= split;
      window -= in_window;
    }
    units = 0;
    for (int q = 0; q < k; ++q) {
      p.req[q].unit_off = units;
      p.req[q].n_pair = pairs_of[q];
      units += tiles_of[q] - pairs_of[q];
    }
  }
  if (units == 0) return TR_OK;
  p.R = k;
  p.n_units = units;
  int smem = 0;
  const int sw = lp_max <= 32 ? 32 : lp_max <= 64 ? 64 : kMaxLp;   // head slot width of this launch
  if (!plan_smem<D>(p, p.n_layer, sw, true, smem))
    return fail(TR_ERR_UNSUPPORTED, "stack kernel: %d layers do not fit shared memory", p.n_layer);
  const int grid = std::min(units, sms);
  if (og)
    return sw == 32 ? launch<D, 32, false, true>(grid, p, smem, st)
         : sw == 64 ? launch<D, 64, false, true>(grid, p, smem, st)
                    : launch<D, kMaxLp, false, true>(grid, p, smem, st);
  return sw == 32 ? launch<D, 32, false>(grid, p, smem, st)
       : sw == 64 ? launch<D, 64, false>(grid, p, smem, st)
                  : launch<D, kMaxLp, false>(grid, p, smem, st);
}

}  // namespace

tr_status tc_score(const tr_model* m, const void* tokens, int64_t n, const int64_t* req_offsets,
                   const void* const* kv, const int32_t* L_u, const int32_t* domain, int R, float* scores,
                   cudaStream_t st) {
  bool fits = true;
  for (int r = 0; r < R; ++r) fits = fits && L_u[r] <= kMaxLp;
  if (!fits) {  // long user sequences: CUDA-core path
    for (int r = 0; r < R; ++r)
      TR_TRY(simt_score(m, tokens, req_offsets[r], req_offsets[r + 1], kv[r], L_u[r], domain[r], scores, st));
    return TR_OK;
  }
  if ((uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "tokens not 16-byte aligned");
  for (int r = 0; r < R; ++r)
    if ((uintptr_t)kv[r] % 16 && L_u[r] > 0 && req_offsets[r + 1] > req_offsets[r])
      return fail(TR_ERR_INVALID_ARG, "kv[%d] is not 16-byte aligned", r);
  return m->desc.D == 128 ? score_launch<128>(m, tokens, req_offsets, kv, L_u, domain, R, scores, st)
                          : score_launch<64>(m, tokens, req_offsets, kv, L_u, domain, R, scores, st);
}

// Candidates of L_t bf16 tokens (the uncompressed-target variant): whether the tensor-core
// stack takes them (L_t a power of two up to 16, so that a candidate's tokens are adjacent
// lanes of one warp, and every request's L_u within the kernel's reach).
bool tc_score_lt_supported(const tr_model* m, int L_t, const int32_t* L_u, int R) {
  if (!(m->desc.dtype == TR_BF16 && tc_stack_supported(m) && L_t >= 1 && L_t <= 16 && (L_t & (L_t - 1)) == 0))
    return false;
  for (int r = 0; r < R; ++r)
    if (L_u[r] > kMaxLp) return false;
  return true;
}

tr_status tc_score_lt(const tr_model* m, const void* tokens, int L_t, const int64_t* req_offsets,
                      const void* const* kv, const int32_t* L_u, const int32_t* domain, int R, float* scores,
                      cudaStream_t st) {
  if ((uintptr_t)tokens % 16) return fail(TR_ERR_INVALID_ARG, "tokens not 16-byte aligned");
  for (int r = 0; r < R; ++r)
    if ((uintptr_t)kv[r] % 16 && L_u[r] > 0 && req_offsets[r + 1] > req_offsets[r])
      return fail(TR_ERR_INVALID_ARG, "kv[%d] is not 16-byte aligned", r);
  return m->desc.D == 128 ? score_launch<128>(m, tokens, req_offsets, kv, L_u, domain, R, scores, st, L_t)
                          : score_launch<64>(m, tokens, req_offsets, kv, L_u, domain, R, scores, st, L_t);
}

bool tc_prefill_supported(const tr_model* m, int L_u) { return tc_stack_supported(m) && L_u <= kMaxLp; }

// User sides of R requests through the same kernel: one CTA per request (with L_u > 0), the
// request's user tokens as its tile.
tr_status tc_prefill_batch(const tr_model* m, const float* const* user_tokens, const int32_t* L_u,
                           const int32_t* domain, void* const* kv, int R, cudaStream_t st) {
  DeviceState* ds = nullptr;
  TR_TRY(device_state(&ds));
  StackParams p{};
  p.wimg = static_cast<const uint8_t*>(m->tc_stack);
  p.vec = m->tc_vec;
  p.domain_emb = m->domain_emb;
  p.status = ds->status;
  p.n_layer = m->desc.n_layer;
  p.pair = 0;
  int k = 0, lp_max = 0;
  for (int r = 0; r < R; ++r) {
    if (L_u[r] == 0) continue;
    if ((uintptr_t)kv[r] % 16 || (uintptr_t)user_tokens[r] % 16)
      return fail(TR_ERR_INVALID_ARG, "request %d: user_tokens / kv not 16-byte aligned", r);
    p.req[k].kv = static_cast<const uint8_t*>(kv[r]);
    p.req[k].utokens = user_tokens[r];
    p.req[k].cand_off = 0;
    p.req[k].n = L_u[r];
    p.req[k].unit_off = k;
    p.req[k].L_u = L_u[r];
    p.req[k].domain = domain[r];
    p.req[k].n_pair = 0;
    lp_max = std::max(lp_max, round_up16(L_u[r]));
    ++k;
  }
  if (k == 0) return TR_OK;
  p.R = k;
  p.n_units = k;
  int smem = 0;
  const int sw = lp_max <= 32 ? 32 : lp_max <= 64 ? 64 : kMaxLp;   // head slot width of this launch
  const bool fit = m->desc.D == 128 ? plan_smem<128>(p, p.n_layer, sw, false, smem)
                                    : plan_smem<64>(p, p.n_layer, sw, false, smem);
  if (!fit) return fail(TR_ERR_UNSUPPORTED, "stack kernel: %d layers do not fit shared memory", p.n_layer);
  if (m->desc.D == 128)
    return sw == 32 ? launch<128, 32, true>(k, p, smem, st)
         : sw == 64 ? launch<128, 64, true>(k, p, smem, st) : launch<128, kMaxLp, true>(k, p, smem, st);
  return sw == 32 ? launch<64, 32, true>(k, p, smem, st)
       : sw == 64 ? launch<64, 64, true>(k, p, smem, st) : launch<64, kMaxLp, true>(k, p, smem, st);
}

// User side of one request (one CTA).
tr_status tc_prefill(const tr_model* m, const float* user_tokens, int L_u, int domain, void* kv, cudaStream_t st) {
  const int32_t lu = L_u, dm = domain;
  void* kvp = kv;
  return tc_prefill_batch(m, &user_tokens, &lu, &dm, &kvp, 1, st);
}

}  // namespace tr
