// Exact softmax attention core for head_dim 64 on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA computes NQ 128-query tiles of one (problem, head) (NQ = 2 in
// global and register mode; frame mode runs the persistent one-tile kernel of
// attention_frame_persistent.cuh with the same per-step code; the text below
// describes NQ = 2).  Configurations (CoreCfg): SGA adds the subsampled global
// attention terms in the epilogue, KTM reads keys token-major like values,
// RANKS reads the keys and values of several ranks' buffers in turn
// (attn_core_ranks_kernel, query-sharded global attention), PART splits one
// row's keys over two launches (the first leaves its softmax state, the
// second merges it; query-sharded global attention with the all-gather
// overlapped):
//   O = softmax(Q K^T) V   over the problem's L keys.  Q arrives scaled by
//   softmax_scale*log2(e) from the prologue, so scores are in base 2.
// (VGGT-Omega Aggregator explainer, section 3: the frame / global / register
// attention of the alternating-attention block; the kernel is the same for
// the three modes, only the workspace views and the output row map differ.)
//
// Keys are processed in steps of 64.  Every Q tile has two S buffers in
// TMEM, so the tensor core computes S(j+2) while the softmax works on S(j+1).
//
// Warp roles (384 threads, 12 warps; 256 threads for NQ = 1):
//   warp 0       TMA producer: both Q tiles once, then K/V tiles of 64 keys
//                through an 8-stage shared-memory ring (128-byte swizzle, no
//                multicast).
//   warps 1, 2   MMA issuers, one per Q tile (warp 1 also allocates TMEM).
//                One thread can issue a tcgen05.mma only every ~45-50 cycles,
//                so the two tiles' streams go out from two threads.  Per step
//                j a tile's stream is
//                  O_i += P_i(j) [V_j | 1]  (M=128, N=80, K=16 x 4, P from TMEM)
//                  S_i(j+2) = Q_i K_j+2^T   (M=128, N=64, K=16 x 4, Q from TMEM,
//                                            into the S buffer P_i(j) came from)
//                  commit -> S_FULL          (also covers PV(j))
//                in program order, so S(j+2) overwrites P(j) only after PV(j).
//                Q sits in TMEM so that a QK^T product reads only its 2 KB of
//                K from shared memory: with Q read from shared memory too
//                (6 KB per product) those products were bound by shared-memory
//                bandwidth rather than by the tensor core.
//                The B operand of PV is V_j followed by 16 columns of ones
//                (a constant shared-memory tile), so columns 64-79 of O_i
//                accumulate the row sums of P on the tensor core and the
//                softmax threads never add their probabilities up.
//   warp 3       idle.
//   warps 4-11   softmax, one warpgroup per Q tile; thread r owns query row r
//                (= TMEM lane r).  First it copies its row of Q from shared
//                memory into TMEM.  Per step it reads its 64 scores, keeps a
//                running reference max m in fp32, writes P = 2^(s - m) as
//                bf16 over the first 32 columns of the S buffer, and rescales
//                O (head dims and the sum column) in TMEM only when m grows by
//                more than 8 (a factor of 256; below that the stale max is
//                kept, which is exact because O and its sum column always
//                share the same m).  A small share of the exponentials runs on
//                the FMA pipe (a cubic for 2^f after an exponent split), the
//                rest on the MUFU unit.  Seeing S(j) complete also tells the
//                warpgroup that PV(j-2) is complete, so it releases K/V stage
//                j-2 to the producer, and a rescale at step j waits for S(j+1)
//                (issued after PV(j-1)) rather than for a barrier of its own.
//                Epilogue: O[:, 0:64] / O[:, 64] -> bf16 -> out.
//
// The row sum is that of the bf16-rounded P that multiplies V, so numerator
// and denominator see the same rounding.
//
// TMEM (512 columns allocated, 256 for NQ = 1): S buffers of tile i at
// columns 128 i and 128 i + 64, O_i at 128 NQ + 80 i (80 columns), Q_i after
// the O accumulators (32 columns each).  Every
// mbarrier wait is bounded (wait_bounded); on expiry the CTA records
// VGGT_ATTN_ERR_TIMEOUT in the workspace status word, drains what it has in
// flight and exits without writing its output tiles.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

// Extra inputs of subsampled global attention (SGA): the per-row diagonal
// and mean-pair terms the epilogue adds to the attention over the kept keys.
struct SgaParams {
  const uint16_t* q_plane;   // normalised q of every token, [H][N][64] (as the core reads it)
  const uint16_t* k_plane;   // normalised k of every token, [H][N][64]
  const uint16_t* qkv;       // raw qkv [N][3][H][64] (v of the diagonal)
  const float* sums;         // [2][H][64]: sums over the discarded tokens of k (0) and v (1)
  int n_d;                   // number of discarded tokens |D|
  float inv_nd;              // 1 / |D| (0 when D is empty)
  int T, n_special, grid_w, s_h, s_w;
};

struct CoreParams {
  int L;              // queries per problem (and keys, except in SGA)
  int Lk;             // keys per problem
  int H;              // heads
  int B;              // problems
  int out_T;          // tokens per frame of `out`
  int out_group;      // query i of problem b -> out row b*out_T + (i/out_group)*out_T + i%out_group
  uint16_t* out;      // bf16 [.][H][64]
  long long out_elems;  // elements of out (bounds of the debug build's checks)
  int* status;
  unsigned long long timeout_ns;
  SgaParams sga;      // SGA configuration only
  int rank_tokens;    // per-rank key blocks (RANKS configuration): keys per rank,
  int rank_steps;     // and 64-key steps per rank (the last one ragged)
  // Softmax state of row i of head h over part of the keys (PART
  // configurations): part_o[(h L + i) 64 + d] = sum over those keys of
  // 2^(s - m) v_d and part_ml[2 (h L + i)] = {sum of 2^(s - m), m}, m the
  // row's reference max (base-2 scores); part_rows = H L.
  float* part_o;
  float* part_ml;
  long long part_rows;
};

// Keys and values of a query-sharded global attention, one tensor map per
// rank over that rank's own buffers ([L][H][64], this GPU's or a peer's).
constexpr int kMaxRankMaps = 8;
struct RankMaps {
  CUtensorMap k[kMaxRankMaps];
  CUtensorMap v[kMaxRankMaps];
};

namespace core {
constexpr int BM = 128, BN = 64, D = 64;
constexpr int Q_BYTES = BM * D * 2;                    // 16 KB query tile
constexpr int KV_BYTES = BN * D * 2;                   // 8 KB key or value tile
constexpr float RESCALE_THRESHOLD = 8.0f;              // log2 units
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
// PV has N = 80: the 64 head dims of V, then 16 columns of ones whose
// products are the row sums of P (every one of columns 64-79 holds it).
constexpr int NV = D + 16;
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, NV, 0, 1);  // V is MN-major (head dim contiguous)
// Exponentials of score pair q (0..31 in a row of a step) run on the FMA pipe
// when bit (q % 8) of this mask is set, on the MUFU unit otherwise.
constexpr uint32_t POLY_PAIR_MASK = 0x80u;
}  // namespace core

// Per-CTA shape of the kernel.  NQ = 2: two 128-query tiles share every K/V
// tile (one CTA per SM; global and register mode, whose key loops are long).
// NQ = 1: one tile per CTA and two CTAs per SM, one launch-time CTA per tile.
// Frame mode (17 key steps per tile) runs the persistent form of the NQ = 1
// shape instead (attention_frame_persistent.cuh): its CTAs take tile after
// tile and start the next tile's products during the last one's epilogue,
// 2 % faster on the 500-frame workload.
template <int NQ_, bool SGA_ = false, bool KTM_ = false, bool RANKS_ = false, int PART_ = 0>
struct CoreCfg {
  static constexpr int NQ = NQ_;
  static constexpr bool SGA = SGA_;   // subsampled global attention epilogue
  // Keys token-major, [Lk][H][64] like the values (query-sharded global mode:
  // the keys all ranks gathered), instead of one [B*Lk][64] plane per head.
  static constexpr bool KTM = KTM_;
  // Keys in per-rank blocks read from each rank's buffers (RankMaps); every
  // block starts a new 64-key step and its last step is masked to its length.
  static constexpr bool RANKS = RANKS_;
  static_assert(!RANKS_ || KTM_, "rank blocks are token-major");
  // Epilogue: 0 writes softmax(Q K^T) V as bf16; 1 writes the rows' softmax
  // state over this launch's keys (CoreParams::part_*) instead; 2 merges that
  // state with its own before writing bf16, so that two launches over
  // disjoint key sets give the attention over their union.
  static constexpr int PART = PART_;
  static_assert(PART_ >= 0 && PART_ <= 2 && !(SGA_ && PART_), "epilogue configuration");
  static constexpr int CTAS_PER_SM = NQ_ == 2 ? 1 : 2;
  static constexpr int STAGES = NQ_ == 2 ? 8 : 5;
  static constexpr int OFF_Q = 0;                                  // NQ tiles
  static constexpr int OFF_K = OFF_Q + NQ * core::Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * core::KV_BYTES;
  static constexpr int OFF_ONES = OFF_V + STAGES * core::KV_BYTES; // 64 x 64 bf16 ones: the PV product's extra columns
  static constexpr int OFF_BAR = OFF_ONES + core::KV_BYTES;
  enum {
    BAR_Q = 0,
    BAR_KV_FULL = 1,
    BAR_KV_EMPTY = BAR_KV_FULL + STAGES,
    BAR_S_FULL = BAR_KV_EMPTY + STAGES,   // [tile][buffer]
    BAR_P_FULL = BAR_S_FULL + NQ * 2,     // [tile][buffer]
    BAR_PV_DONE = BAR_P_FULL + NQ * 2,    // [tile]
    BAR_O_FINAL = BAR_PV_DONE + NQ,       // [tile]
    BAR_Q_TMEM = BAR_O_FINAL + NQ,        // [tile]: Q copied into TMEM
    BAR_DRAIN = BAR_Q_TMEM + NQ,          // [issuer]
    N_BARS = BAR_DRAIN + NQ
  };
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;          // tmem slot, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;           // slack to align the base to 1024 B
  static constexpr int THREADS = 128 * (1 + NQ);                 // producer/issuer warpgroup + one per tile
  // TMEM per tile i: S buffers at 128 i and 128 i + 64, O (80 columns) at
  // COL_O + 80 i, Q (64 dims as bf16 pairs) at COL_Q + 32 i.
  static constexpr uint32_t TMEM_COLS = NQ == 2 ? 512 : 256;
  static constexpr uint32_t COL_O = 128 * NQ;
  static constexpr uint32_t COL_Q = COL_O + core::NV * NQ;
  static_assert(COL_Q + 32 * NQ <= TMEM_COLS, "TMEM layout");
  // Register split (setmaxnreg): warpgroup 0 gives registers back, the
  // softmax warpgroups take them; the sum never exceeds the launch allocation
  // (the host checks the compiled register count before every launch).
  static constexpr int REGS_AT_LAUNCH = NQ == 2 ? 168 : 128;
  static constexpr int REGS_PRODUCER = 56;
  static constexpr int REGS_SOFTMAX = NQ == 2 ? 224 : 200;
  static_assert(REGS_PRODUCER * 128 + REGS_SOFTMAX * 128 * NQ <= REGS_AT_LAUNCH * THREADS, "register split too large");
  static_assert(REGS_AT_LAUNCH * THREADS * CTAS_PER_SM <= 65536, "registers per SM");
};

// Local names for a configuration's constants inside the templated roles.
#define VGGT_CORE_CFG_NAMES(C)                                                                          \
  constexpr int NQ = C::NQ, STAGES = C::STAGES;                                                        \
  constexpr int OFF_Q = C::OFF_Q, OFF_K = C::OFF_K, OFF_V = C::OFF_V, OFF_ONES = C::OFF_ONES;          \
  constexpr int OFF_BAR = C::OFF_BAR, OFF_MISC = C::OFF_MISC;                                          \
  constexpr uint32_t TMEM_COLS = C::TMEM_COLS, COL_O = C::COL_O, COL_Q = C::COL_Q;                      \
  constexpr int REGS_SOFTMAX = C::REGS_SOFTMAX, REGS_PRODUCER = C::REGS_PRODUCER;                      \
  constexpr int BAR_Q = C::BAR_Q, BAR_KV_FULL = C::BAR_KV_FULL, BAR_KV_EMPTY = C::BAR_KV_EMPTY;        \
  constexpr int BAR_S_FULL = C::BAR_S_FULL, BAR_P_FULL = C::BAR_P_FULL, BAR_PV_DONE = C::BAR_PV_DONE;  \
  constexpr int BAR_O_FINAL = C::BAR_O_FINAL, BAR_Q_TMEM = C::BAR_Q_TMEM, BAR_DRAIN = C::BAR_DRAIN;    \
  (void)NQ; (void)STAGES; (void)OFF_Q; (void)OFF_K; (void)OFF_V; (void)OFF_ONES; (void)OFF_BAR;         \
  (void)OFF_MISC; (void)TMEM_COLS; (void)COL_O; (void)COL_Q; (void)REGS_SOFTMAX; (void)REGS_PRODUCER;   \
  (void)BAR_Q; (void)BAR_KV_FULL; (void)BAR_KV_EMPTY; (void)BAR_S_FULL; (void)BAR_P_FULL;               \
  (void)BAR_PV_DONE; (void)BAR_O_FINAL; (void)BAR_Q_TMEM; (void)BAR_DRAIN


struct PolyConsts {
  uint64_t shift2, c3, c2, c1, c0;   // each: the same fp32 constant in both halves
};
__device__ __forceinline__ uint64_t dup_f32(float v) {
  const uint64_t u = __float_as_uint(v);
  return u | (u << 32);
}
__device__ __forceinline__ PolyConsts poly_consts() {
  return {dup_f32(12582912.0f), dup_f32(5.517166853e-02f), dup_f32(2.426111251e-01f), dup_f32(6.932609677e-01f),
          dup_f32(9.999280572e-01f)};
}
// 2^x for x <= ~128 on the FMA pipe, two values at once: x = j + f with
// j = round(x) (via the 1.5*2^23 shift), f in [-1/2, 1/2]; 2^f from a cubic
// fitted by minimax in relative error (fit_exp2_poly.py, max rel. error
// 7.5e-5); 2^j added to the exponent field.  x is clamped at -125 so that the
// exponent field never underflows (2^-125 is far below any probability that
// survives bf16 rounding next to the row maximum's 1).
__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& y0, float& y1, const PolyConsts& k) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  float t0, t1, p0, p1;
  asm("{\n\t.reg .b64 rx, rt, rr, rf, rp;\n\t"
      "mov.b64 rx, {%4, %5};\n\t"
      "add.rn.f32x2 rt, rx, %6;\n\t"
      "sub.rn.f32x2 rr, rt, %6;\n\t"
      "sub.rn.f32x2 rf, rx, rr;\n\t"
      "fma.rn.f32x2 rp, %7, rf, %8;\n\t"
      "fma.rn.f32x2 rp, rp, rf, %9;\n\t"
      "fma.rn.f32x2 rp, rp, rf, %10;\n\t"
      "mov.b64 {%0, %1}, rt;\n\t"
      "mov.b64 {%2, %3}, rp;\n\t}"
      : "=f"(t0), "=f"(t1), "=f"(p0), "=f"(p1)
      : "f"(x0), "f"(x1), "l"(k.shift2), "l"(k.c3), "l"(k.c2), "l"(k.c1), "l"(k.c0));
  // bits(2^f) + round(x) << 23; the low mantissa bits of t hold round(x) and
  // the multiply by 2^23 drops the rest of t's bits out of the word.
  uint32_t b0, b1;
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(b0) : "r"(__float_as_uint(t0)), "r"(__float_as_uint(p0)));
  asm("mad.lo.u32 %0, %1, 8388608, %2;" : "=r"(b1) : "r"(__float_as_uint(t1)), "r"(__float_as_uint(p1)));
  y0 = __uint_as_float(b0);
  y1 = __uint_as_float(b1);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (a0, a1) + (b0, b1) as one packed instruction.
__device__ __forceinline__ void add_x2(float a0, float a1, float b0, float b1, float& d0, float& d1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// 32 lanes x 1 column load / store.
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}

// 32 lanes x 16 columns store.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Subsampled global attention (AVGGT article, section B, point 2): query i
// also sees its own key when that key was discarded (the diagonal) and the
// mean of the discarded keys/values counted n_i = |D| - [i discarded] times.
// Folds both into the row's accumulator `o` (64 head dims) and row sum `osum`,
// which are relative to the reference max m (base-2 scores: q is pre-scaled).
__device__ __forceinline__ float dot_bf16_row(const uint16_t* a, const float* b_f32, const uint16_t* b_bf16) {
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 w = a4[k];
    const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(wd[e] << 16), hi = __uint_as_float(wd[e] & 0xFFFF0000u);
      const int d = 8 * k + 2 * e;
      float blo, bhi;
      if (b_f32) {
        blo = b_f32[d];
        bhi = b_f32[d + 1];
      } else {
        const uint32_t bw = reinterpret_cast<const uint32_t*>(b_bf16)[d >> 1];
        blo = __uint_as_float(bw << 16);
        bhi = __uint_as_float(bw & 0xFFFF0000u);
      }
      acc[e] += lo * blo + hi * bhi;
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
}

__device__ __forceinline__ void sga_extra_terms(const CoreParams& p, int h, int i, float m, uint32_t (&o)[2][32],
                                                uint32_t& osum) {
  const SgaParams& g = p.sga;
  const int t = i % g.T;
  bool kept = t < g.n_special;
  if (!kept) {
    const int pp = t - g.n_special;
    const int prow = pp / g.grid_w, pcol = pp - prow * g.grid_w;
    kept = (prow % g.s_h == 0) && (pcol % g.s_w == 0);
  }
  const bool diag = !kept;
  const int n_mean = g.n_d - (diag ? 1 : 0);
  if (!diag && n_mean <= 0) return;
  const uint16_t* q = g.q_plane + (static_cast<size_t>(h) * p.L + i) * 64;
  const float* ksum = g.sums + h * 64;
  const float* vsum = g.sums + (p.H + h) * 64;
  float m2 = m, s_d = 0.f, s_m = 0.f, lw = 0.f;
  if (diag) {
    s_d = dot_bf16_row(q, nullptr, g.k_plane + (static_cast<size_t>(h) * p.L + i) * 64);
    m2 = fmaxf(m2, s_d);
  }
  if (n_mean > 0) {
    s_m = dot_bf16_row(q, ksum, nullptr) * g.inv_nd;
    lw = log2f(static_cast<float>(n_mean));
    m2 = fmaxf(m2, s_m + lw);
  }
  const float a = exp2f(m - m2);
  const float pd = diag ? exp2f(s_d - m2) : 0.f;
  const float pm = n_mean > 0 ? exp2f(s_m + lw - m2) * g.inv_nd : 0.f;   // weight of the mean pair, per unit of vsum
  const uint16_t* v = g.qkv + (static_cast<size_t>(i) * 3 + 2) * p.H * 64 + h * 64;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int d = 32 * c + e;
      const uint32_t vw = reinterpret_cast<const uint32_t*>(v)[d >> 1];
      const float v0 = __uint_as_float(vw << 16), v1 = __uint_as_float(vw & 0xFFFF0000u);
      o[c][e] = __float_as_uint(__uint_as_float(o[c][e]) * a + pd * v0 + pm * vsum[d]);
      o[c][e + 1] = __float_as_uint(__uint_as_float(o[c][e + 1]) * a + pd * v1 + pm * vsum[d + 1]);
    }
  }
  osum = __float_as_uint(__uint_as_float(osum) * a + pd + pm * static_cast<float>(g.n_d));
}

// Softmax warpgroup role: warps 4-7 own Q tile 0 (TILE = 0), warps 8-11 Q
// tile 1 (TILE = 1).
template <class C, int TILE>
__device__ __forceinline__ void softmax_role(const CoreParams& p, const uint8_t* smem, uint32_t tmem, uint32_t bar0,
                                             volatile int* abort_flag, int h, int b, int q0, int n_kv, int warp,
                                             int lane) {
  using namespace core;
  VGGT_CORE_CFG_NAMES(C);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int tile = TILE;
  const int quarter = warp & 3;              // TMEM lane quarter this warp may access
  const int row = quarter * 32 + lane;       // query row of this thread in its tile
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t s_base = tmem + lane_base + tile * 2 * BN;
  const uint32_t o_addr = tmem + lane_base + COL_O + tile * NV;
  const PolyConsts pc = poly_consts();
  float m_run = -INFINITY;
  // Q tile -> TMEM (A operand of the QK^T products: row r in lane r, dims
  // (2c, 2c+1) in column c), so that those products read only K from shared
  // memory.  The tile sits in shared memory with the 128-byte swizzle: 16-byte
  // chunk c of row r is stored at chunk c ^ (r % 8).
  bool ok = wait_bounded(bar(BAR_Q), 0, abort_flag, p.status, p.timeout_ns, 0x330u | tile);
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) return;
  {
    const uint4* qrow = reinterpret_cast<const uint4*>(smem + OFF_Q + tile * Q_BYTES + row * 128);
    uint32_t qr[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = qrow[c ^ (row & 7)];
      qr[4 * c] = v.x;
      qr[4 * c + 1] = v.y;
      qr[4 * c + 2] = v.z;
      qr[4 * c + 3] = v.w;
    }
    tmem_st32(tmem + lane_base + COL_Q + tile * (D / 2), qr);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar(BAR_Q_TMEM + tile));
  }
  int jr = 0;   // step inside the current rank block (RANKS configuration)
  (void)jr;
  for (int j = 0; j < n_kv; ++j) {
    const int buf = j & 1;
    const uint32_t s_addr = s_base + buf * BN;
    ok = wait_bounded(bar(BAR_S_FULL + tile * 2 + buf), (j >> 1) & 1, abort_flag, p.status, p.timeout_ns,
                      0x300u | tile);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    // S(j) completing means PV(j-2) (issued before it by the same thread)
    // has completed too: K/V stage j-2 is no longer read by this tile.
    if (j >= 2 && (threadIdx.x & 127) == 0) mbar_arrive(bar(BAR_KV_EMPTY + (j - 2) % STAGES));
    tc_fence_after();
    uint32_t sr[2][32];
    tmem_ld32(s_addr, sr[0]);
    tmem_ld32(s_addr + 32, sr[1]);
    tmem_wait_ld();
    // keys of this step that exist (>= BN except on the last step, or on each
    // rank block's last step)
    int valid;
    if constexpr (C::RANKS) {
      valid = p.rank_tokens - jr * BN;
      if (++jr == p.rank_steps) jr = 0;
    } else {
      valid = p.Lk - j * BN;
    }
    if (valid < BN) {                        // last step only (uniform branch)
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c * 32 + e >= valid) sr[c][e] = __float_as_uint(-INFINITY);
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      mx0 = max3f(mx0, __uint_as_float(sr[0][e]), __uint_as_float(sr[0][e + 1]));
      mx1 = max3f(mx1, __uint_as_float(sr[1][e]), __uint_as_float(sr[1][e + 1]));
    }
    const float tile_max = fmaxf(mx0, mx1);
    // Move the reference max on the first step, or when it grows by more
    // than the threshold.
    const bool move = (j == 0) || (tile_max > m_run + RESCALE_THRESHOLD);
    float alpha = 1.f;
    if (move) {
      alpha = (j == 0) ? 0.f : ex2_approx(m_run - tile_max);
      m_run = tile_max;
    }
    const float neg_m = -m_run;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float x0, x1, p0, p1;
        add_x2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]), neg_m, neg_m, x0, x1);
        const int pair = (c * 32 + e) >> 1;
        if ((POLY_PAIR_MASK >> (pair & 7)) & 1u) {
          exp2_poly_x2(x0, x1, p0, p1, pc);
        } else {
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        pk[e >> 1] = pack_bf16x2(p0, p1);
      }
      // P (64 keys -> 32 columns) overwrites the first 32 columns of this S buffer.
      tmem_st16(s_addr + c * 16, pk);
    }
    // O must be rescaled before PV(j) accumulates into it, and after PV(j-1)
    // has: PV(j-2) is known complete (S(j) was issued after it and has
    // completed), so PV_DONE is at most one phase behind.  Warp-uniform:
    // tcgen05.ld/st are warp-collective.
    if (__any_sync(0xffffffffu, move && j > 0)) {
      // PV(j-1) must be complete: S(j+1) was issued after it, so its
      // completion says so; past the last S, PV_DONE (committed only when no
      // S follows a PV, first for PV(n_kv-2)) does.
      ok = (j + 1 < n_kv)
               ? wait_bounded(bar(BAR_S_FULL + tile * 2 + ((j + 1) & 1)), ((j + 1) >> 1) & 1, abort_flag, p.status,
                              p.timeout_ns, 0x310u | tile)
               : wait_bounded(bar(BAR_PV_DONE + tile), 0, abort_flag, p.status, p.timeout_ns, 0x318u | tile);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t orr[2][32], osum;
      tmem_ld32(o_addr, orr[0]);
      tmem_ld32(o_addr + 32, orr[1]);
      tmem_ld1(o_addr + D, osum);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) orr[c][e] = __float_as_uint(__uint_as_float(orr[c][e]) * alpha);
      osum = __float_as_uint(__uint_as_float(osum) * alpha);
      tmem_st32(o_addr, orr[0]);
      tmem_st32(o_addr + 32, orr[1]);
      tmem_st1(o_addr + D, osum);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar(BAR_P_FULL + tile * 2 + buf));
  }
  if (ok) {
    ok = wait_bounded(bar(BAR_O_FINAL + tile), 0, abort_flag, p.status, p.timeout_ns, 0x320u | tile);
    ok = __all_sync(0xffffffffu, ok);
  }
  if (ok) {
    tc_fence_after();
    uint32_t orr[2][32], osum;
    tmem_ld32(o_addr, orr[0]);
    tmem_ld32(o_addr + 32, orr[1]);
    tmem_ld1(o_addr + D, osum);
    tmem_wait_ld();
    const int i = q0 + tile * BM + row;
    if (C::PART == 1 && i < p.L) {
      const long long pr = static_cast<long long>(h) * p.L + i;
      if (VGGT_DBG_BOUNDS(pr < p.part_rows, p.status, 0x930u)) {
        float4* dst = reinterpret_cast<float4*>(p.part_o + pr * D);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[c * 8 + v] = make_float4(__uint_as_float(orr[c][4 * v]), __uint_as_float(orr[c][4 * v + 1]),
                                         __uint_as_float(orr[c][4 * v + 2]), __uint_as_float(orr[c][4 * v + 3]));
        reinterpret_cast<float2*>(p.part_ml)[pr] = make_float2(__uint_as_float(osum), m_run);
      }
    } else if (i < p.L) {
      if constexpr (C::SGA) sga_extra_terms(p, h, i, m_run, orr, osum);
      if constexpr (C::PART == 2) {
        // The other launch's state over its keys, both relative to their own
        // reference max: scale each to the larger one and add.
        const long long pr = static_cast<long long>(h) * p.L + i;
        if (VGGT_DBG_BOUNDS(pr < p.part_rows, p.status, 0x938u)) {
          const float2 ml = reinterpret_cast<const float2*>(p.part_ml)[pr];
          const float m = fmaxf(m_run, ml.y);
          const float a_own = ex2_approx(m_run - m), a_part = ex2_approx(ml.y - m);
          const float4* src = reinterpret_cast<const float4*>(p.part_o + pr * D);
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 o1 = src[c * 8 + v];
              uint32_t* o = &orr[c][4 * v];
              o[0] = __float_as_uint(__uint_as_float(o[0]) * a_own + o1.x * a_part);
              o[1] = __float_as_uint(__uint_as_float(o[1]) * a_own + o1.y * a_part);
              o[2] = __float_as_uint(__uint_as_float(o[2]) * a_own + o1.z * a_part);
              o[3] = __float_as_uint(__uint_as_float(o[3]) * a_own + o1.w * a_part);
            }
          osum = __float_as_uint(__uint_as_float(osum) * a_own + ml.x * a_part);
        }
      }
      const float inv = 1.f / __uint_as_float(osum);
      const long long out_row = static_cast<long long>(b) * p.out_T +
                                static_cast<long long>(i / p.out_group) * p.out_T + (i % p.out_group);
      uint4* dst = reinterpret_cast<uint4*>(p.out + (out_row * p.H + h) * D);
      const bool in_bounds = VGGT_DBG_BOUNDS((out_row * p.H + h + 1) * D <= p.out_elems, p.status, 0x900u);
#pragma unroll
      for (int c = 0; c < 2 && in_bounds; ++c) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          const uint32_t* o = &orr[c][v * 8];
          w.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
          dst[c * 4 + v] = w;
        }
      }
    }
  }
}

// Body of the core kernels: k_maps / v_maps hold one tensor map (or, for the
// RANKS configuration, one per rank).
template <class C>
__device__ __forceinline__ void attn_core_body(const CUtensorMap* q_map, const CUtensorMap* k_maps,
                                               const CUtensorMap* v_maps, const CoreParams& p) {
  using namespace core;
  VGGT_CORE_CFG_NAMES(C);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = blockIdx.x * (NQ * BM);
  const int n_tiles = (NQ > 1 && q0 + BM < p.L) ? 2 : 1;   // the second Q tile may lie past the end
  const int n_kv = (p.Lk + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), n_tiles);   // one arrival per Q tile's softmax warpgroup
    }
    for (int i = 0; i < NQ; ++i) {
      for (int buf = 0; buf < 2; ++buf) {
        mbar_init(bar(BAR_S_FULL + i * 2 + buf), 1);
        mbar_init(bar(BAR_P_FULL + i * 2 + buf), 128);
      }
      mbar_init(bar(BAR_PV_DONE + i), 1);
      mbar_init(bar(BAR_O_FINAL + i), 1);
      mbar_init(bar(BAR_Q_TMEM + i), 128);
      mbar_init(bar(BAR_DRAIN + i), 1);
    }
    fence_mbar_init();
    *abort_flag = status_is_set(p.status) ? 1 : 0;  // another CTA already failed: skip the work
    tma_prefetch_desc(q_map);
    tma_prefetch_desc(&k_maps[0]);
    tma_prefetch_desc(&v_maps[0]);
  }
  for (int e = threadIdx.x; e < KV_BYTES / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(smem + OFF_ONES)[e] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == 1) {
    tmem_alloc(smem_addr(const_cast<uint32_t*>(tmem_slot)), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool skip = *abort_flag != 0;

  if (warp >= 4) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(REGS_SOFTMAX));
    // One copy of the softmax per tile, with the tile index a compile-time
    // constant in each (measured 3-8% faster than one copy shared by both).
    if (!skip && ((warp >> 2) - 1) < n_tiles) {
      if (warp < 8)
        softmax_role<C, 0>(p, smem, tmem, bar0, abort_flag, h, b, q0, n_kv, warp, lane);
      else if constexpr (NQ > 1)
        softmax_role<C, 1>(p, smem, tmem, bar0, abort_flag, h, b, q0, n_kv, warp, lane);
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PRODUCER));
  }
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !skip) {
      int issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      mbar_arrive_expect_tx(bar(BAR_Q), n_tiles * Q_BYTES);
      for (int i = 0; i < n_tiles; ++i)
        tma_load_3d(sbase + OFF_Q + i * Q_BYTES, q_map, bar(BAR_Q), 0, q0 + i * BM, h * p.B + b);
      bool ok = true;
      int kr = 0, jr = 0;   // rank block and step inside it (RANKS configuration)
      (void)kr;
      (void)jr;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % STAGES;
        if (j >= STAGES) {
          ok = wait_bounded(bar(BAR_KV_EMPTY + st), ((j / STAGES) - 1) & 1, abort_flag, p.status, p.timeout_ns,
                            0x100u | st);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bar(BAR_KV_FULL + st), 2 * KV_BYTES);
        if constexpr (C::RANKS) {
          tma_load_4d(sbase + OFF_K + st * KV_BYTES, &k_maps[kr], bar(BAR_KV_FULL + st), 0, h, jr * BN, 0);
          tma_load_4d(sbase + OFF_V + st * KV_BYTES, &v_maps[kr], bar(BAR_KV_FULL + st), 0, h, jr * BN, 0);
          if (++jr == p.rank_steps) {
            jr = 0;
            ++kr;
          }
        } else {
          if constexpr (C::KTM)
            tma_load_4d(sbase + OFF_K + st * KV_BYTES, &k_maps[0], bar(BAR_KV_FULL + st), 0, h, j * BN, b);
          else
            tma_load_3d(sbase + OFF_K + st * KV_BYTES, &k_maps[0], bar(BAR_KV_FULL + st), 0, j * BN, h * p.B + b);
          tma_load_4d(sbase + OFF_V + st * KV_BYTES, &v_maps[0], bar(BAR_KV_FULL + st), 0, h, j * BN, b);
        }
        ++issued[st];
      }
      if (!ok) {
        // Drain: the last load issued into every stage (and Q) must land
        // before this CTA's shared memory is released.
        wait_drain(bar(BAR_Q), 0, p.timeout_ns);
        for (int st = 0; st < STAGES; ++st)
          if (issued[st] > 0) wait_drain(bar(BAR_KV_FULL + st), (issued[st] - 1) & 1, p.timeout_ns);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    const int i = warp - 1;
    if (lane == 0 && !skip && i < n_tiles) {
      // Descriptors differ only in their start-address field (address >> 4).
      const uint64_t dk = smem_desc_sw128(sbase + OFF_K, 16, 1024);
      const uint32_t t_s = tmem + i * 2 * BN, t_o = tmem + COL_O + i * NV;
      const uint32_t t_q = tmem + COL_Q + i * (D / 2);
      auto issue_s = [&](int jj) {    // S(jj) into buffer jj % 2 from key stage jj % STAGES, Q from TMEM
        const uint64_t k = dk + (jj % STAGES) * (KV_BYTES >> 4);
        const uint32_t d = t_s + (jj & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ts(d, t_q + kk * 8, k + 2 * kk, IDESC_QK, kk > 0);
      };
      auto issue_pv = [&](int jj) {   // O += P(jj) V(jj), P in buffer jj % 2 (64 keys = 32 columns)
        // Second MN atom (columns 64-79) = the ones tile: LBO is its distance
        // from this stage's V tile.
        const uint32_t v_addr = sbase + OFF_V + (jj % STAGES) * KV_BYTES;
        const uint64_t v = smem_desc_sw128(v_addr, sbase + OFF_ONES - v_addr, 1024);
        const uint32_t a = t_s + (jj & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(t_o, a + kk * 8, v + kk * (2048 >> 4), IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bounded(bar(BAR_Q_TMEM + i), 0, abort_flag, p.status, p.timeout_ns, 0x200u);
      // Stagger the two tiles: tile 1 starts once tile 0's first softmax step
      // is done, so the two softmax warpgroups run out of phase.
      if (ok && i == 1) ok = wait_bounded(bar(BAR_P_FULL + 0), 0, abort_flag, p.status, p.timeout_ns, 0x2F0u);
      for (int jj = 0; jj < 2 && jj < n_kv && ok; ++jj) {
        ok = wait_bounded(bar(BAR_KV_FULL + jj), 0, abort_flag, p.status, p.timeout_ns, 0x210u | jj);
        if (!ok) break;
        tc_fence_after();
        issue_s(jj);
        tc_commit(bar(BAR_S_FULL + i * 2 + jj));
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int buf = j & 1;
        const int jn = j + 2;
        // K/V of step j+2 first (normally long resident), so that nothing
        // but the MMAs sits between P(j) arriving and S(j+2) being issued.
        if (jn < n_kv) {
          ok = wait_bounded(bar(BAR_KV_FULL + (jn % STAGES)), (jn / STAGES) & 1, abort_flag, p.status,
                            p.timeout_ns, 0x230u | i);
          if (!ok) break;
        }
        ok = wait_bounded(bar(BAR_P_FULL + i * 2 + buf), (j >> 1) & 1, abort_flag, p.status, p.timeout_ns,
                          0x220u | i);
        if (!ok) break;
        tc_fence_after();
        issue_pv(j);
        if (jn < n_kv) {
          issue_s(jn);
          tc_commit(bar(BAR_S_FULL + i * 2 + buf));   // also covers PV(j)
        } else {
          tc_commit(bar(BAR_PV_DONE + i));
          if (j == n_kv - 1) tc_commit(bar(BAR_O_FINAL + i));
        }
      }
      if (!ok) {  // let every MMA already issued finish before TMEM is released
        tc_commit(bar(BAR_DRAIN + i));
        wait_drain(bar(BAR_DRAIN + i), 0, p.timeout_ns);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Fault-path self-test: one bounded wait on a barrier nobody arrives at.
template <class C>
__global__ void __launch_bounds__(C::THREADS, C::CTAS_PER_SM)
    attn_core_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const CoreParams p) {
  attn_core_body<C>(&tmap_q, &tmap_k, &tmap_v, p);
}

// Query-sharded global attention with the keys and values of every rank read
// in place (RANKS configuration; at most kMaxRankMaps ranks).
template <class C>
__global__ void __launch_bounds__(C::THREADS, C::CTAS_PER_SM)
    attn_core_ranks_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ RankMaps maps,
                           const CoreParams p) {
  attn_core_body<C>(&tmap_q, maps.k, maps.v, p);
}

__global__ void selftest_timeout_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_storage;
  const uint32_t b = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    abort_storage = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    wait_bounded(b, 0, &abort_storage, status, timeout_ns, 0xF00u);
  }
}

}  // namespace vggt
