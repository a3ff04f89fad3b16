// Exact softmax attention core for head_dim 64 on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA computes two 128-query tiles (256 queries) of one (problem, head):
//   O = softmax(Q K^T) V   over the problem's L keys.  Q arrives scaled by
//   softmax_scale*log2(e) from the prologue, so scores are in base 2.
// (VGGT-Omega Aggregator explainer, section 3: the frame / global / register
// attention of the alternating-attention block; the kernel is the same for
// the three modes, only the workspace views and the output row map differ.)
//
// Warp roles (640 threads, 20 warps):
//   warp 0       TMA producer: both Q tiles once, then K/V tiles of 128 keys
//                through a 4-stage shared-memory ring (128-byte swizzle, no
//                multicast).
//   warps 1, 2   MMA issuers, one per Q tile (warp 1 also allocates TMEM).
//                One thread can issue a tcgen05.mma only every ~45-50 cycles
//                whatever its size, and the N=64 products below need 32, so
//                the two tiles' streams are issued by two threads:
//                  S_i = Q_i K_j^T      (M=128, N=128, K=16 x 4, fp32 in TMEM)
//                  O_ih += P_ih V_jh    (M=128, N=64,  K=16 x 4 per key half h)
//                in the order PV_i(j-1), S_i(j) (program order of one thread,
//                so the commit that publishes S_i(j) also proves that PV_i(j-1)
//                has finished).  Tile 1 starts once tile 0's first softmax is
//                done, so the two tiles' softmax phases alternate.
//   warp 3       idle.
//   warps 4-19   softmax, four warpgroups: (tile 0, keys 0-63 of every key
//                tile), (tile 0, keys 64-127), (tile 1, keys 0-63), (tile 1,
//                keys 64-127).  Each warpgroup runs its own online softmax over
//                its half of the keys -- running reference max m, sum l and
//                accumulator O_ih of its own -- so the two halves of a row never
//                synchronise inside the key loop; they are merged once at the
//                end: m = max(m_0, m_1), O = sum_h 2^(m_h - m) O_ih and
//                l = sum_h 2^(m_h - m) l_h.  Thread r of a warpgroup owns query
//                row r (= TMEM lane r).  Per key tile it reads its 64 scores
//                from TMEM, writes P = 2^(s - m) as bf16 over the first 32 of
//                its S columns, and rescales O_ih only when m grows by more than
//                8 (a factor of 256; below that the stale max is kept, which is
//                exact because O_ih and l_h always share the same m).  A small
//                share of the exponentials runs on the FMA pipe (a cubic for
//                2^f after an exponent split), the rest on the MUFU unit.

// TMEM (512 columns): tile i owns columns 256 i .. 256 i + 255: S/P at +0,
// O_i0 at +128, O_i1 at +192.  Every mbarrier wait is bounded
// (wait_bounded); on expiry the CTA records VGGT_ATTN_ERR_TIMEOUT in the
// workspace status word, drains what it has in flight and exits without
// writing its output tiles.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

struct CoreParams {
  int L;              // keys (and queries) per problem
  int H;              // heads
  int B;              // problems
  int out_T;          // tokens per frame of `out`
  int out_group;      // query i of problem b -> out row b*out_T + (i/out_group)*out_T + i%out_group
  uint16_t* out;      // bf16 [.][H][64]
  int* status;
  unsigned long long timeout_ns;
};

namespace core {
constexpr int BM = 128, BN = 128, D = 64, STAGES = 4, NQ = 2;
constexpr int HALF = BN / 2;                           // key columns per softmax warpgroup
constexpr int TILE_BYTES = BM * D * 2;                 // 16 KB (Q, K or V tile)
constexpr int OFF_Q = 0;                               // NQ tiles
constexpr int OFF_K = OFF_Q + NQ * TILE_BYTES;
constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr int OFF_XCHG = OFF_V + STAGES * TILE_BYTES;  // float2 [NQ][2 halves][BM]: final (m, l) of each half
constexpr int OFF_BAR = OFF_XCHG + NQ * 2 * BM * 8;
enum {
  BAR_Q = 0,
  BAR_KV_FULL = 1,
  BAR_KV_EMPTY = BAR_KV_FULL + STAGES,
  BAR_S_FULL = BAR_KV_EMPTY + STAGES,
  BAR_P_FULL = BAR_S_FULL + NQ,
  BAR_O_FINAL = BAR_P_FULL + NQ,
  BAR_XCHG = BAR_O_FINAL + NQ,        // one per (tile, lane quarter): the two halves' warps
  BAR_DRAIN = BAR_XCHG + NQ * 4,     // one per MMA issuer
  N_BARS = BAR_DRAIN + NQ
};
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;         // tmem slot, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;          // slack to align the base to 1024 B
constexpr int THREADS = 640;
constexpr bool PERSISTENT = false;                  // grid: one CTA per SM over all units, or one CTA per unit
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TILE_COLS = 256;                    // TMEM columns per Q tile
constexpr uint32_t COL_O = 128;                       // O_i0 offset inside a tile's columns (O_i1 at +64)
constexpr float RESCALE_THRESHOLD = 8.0f;              // log2 units
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);  // V is MN-major (head dim contiguous)
// Exponentials of score pair q (0..31 in a half row) run on the FMA pipe when
// bit (q % 8) of this mask is set, on the MUFU unit otherwise.
constexpr uint32_t POLY_PAIR_MASK = 0x80u;
// Register split (setmaxnreg): the block launches with REGS_AT_LAUNCH per
// thread; warpgroup 0 (TMA + MMA warps) gives registers back, the four softmax
// warpgroups take them.  The sum never exceeds the launch allocation
// (launch_core checks the compiled register count before every launch).
constexpr int REGS_AT_LAUNCH = 96;
constexpr int REGS_PRODUCER = 32;
constexpr int REGS_SOFTMAX = 112;
static_assert(REGS_PRODUCER * 128 + REGS_SOFTMAX * 512 <= REGS_AT_LAUNCH * THREADS, "register split too large");
}  // namespace core

// 2^x for x <= ~128 on the FMA pipe, two values at once: x = j + f with
// j = round(x) (via the 1.5*2^23 shift), f in [-1/2, 1/2]; 2^f from a cubic
// fitted by minimax in relative error (fit_exp2_poly.py, max rel. error
// 7.5e-5); 2^j added to the exponent field.  x is clamped at -125 so that the
// exponent field never underflows (2^-125 is far below any probability that
// survives bf16 rounding next to the row maximum's 1).
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

// 32 lanes x 16 columns store.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Softmax role of one warp: `tile` (Q tile), `half` (key columns 64*half ..
// 64*half+63 of every key tile), `quarter` (TMEM lanes / rows 32*quarter ..).
__device__ __forceinline__ void softmax_role(const CoreParams& p, uint32_t tmem, uint32_t bar0, float2* xchg,
                                             volatile int* abort_flag, int h, int b, int q0, int n_kv, int warp,
                                             int lane) {
  using namespace core;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int g = (warp >> 2) - 1;             // softmax warpgroup 0..3
  const int tile = g >> 1, half = g & 1;
  const int quarter = warp & 3;              // TMEM lane quarter this warp may access
  const int row = quarter * 32 + lane;       // query row of this thread in its tile
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t t_base = tmem + lane_base + tile * TILE_COLS;
  const uint32_t s_addr = t_base + half * HALF;
  const uint32_t o_addr = t_base + COL_O + half * D;
  float m_run = -INFINITY, l_run = 0.f;
  const PolyConsts pc = poly_consts();
  bool ok = true;
  for (int j = 0; j < n_kv; ++j) {
    ok = wait_bounded(bar(BAR_S_FULL + tile), j & 1, abort_flag, p.status, p.timeout_ns, 0x300u | tile);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    uint32_t sr[2][32];
    tmem_ld32(s_addr, sr[0]);
    tmem_ld32(s_addr + 32, sr[1]);
    tmem_wait_ld();
    const int valid = p.L - j * BN - half * HALF;   // keys of this half tile that exist
    if (valid < HALF) {                              // last key tile only (uniform branch)
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
    // Move the reference max on the first tile, or when it grows by more
    // than the threshold.  A half with no valid key yet keeps m = -inf.
    const bool move = (j == 0) || (tile_max > m_run + RESCALE_THRESHOLD);
    float alpha = 1.f;
    if (move) {
      alpha = (j == 0 || m_run == -INFINITY) ? 0.f : ex2_approx(m_run - tile_max);
      m_run = tile_max;
    }
    const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
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
        if (e & 2) {
          add_x2(acc2, acc3, p0, p1, acc2, acc3);
        } else {
          add_x2(acc0, acc1, p0, p1, acc0, acc1);
        }
        pk[e >> 1] = pack_bf16x2(p0, p1);
      }
      // P of this half (64 keys -> 32 columns) overwrites the first 32 of the
      // half's own 64 S columns: the other half's S is never touched.
      tmem_st16(s_addr + c * 16, pk);
    }
    l_run = l_run * alpha + ((acc0 + acc1) + (acc2 + acc3));
    // O_ih must be rescaled before PV_ih(j) accumulates into it.  PV(j-1) is
    // complete: the commit that published S_i(j) came after it.
    // Warp-uniform: tcgen05.ld/st are warp-collective.
    if (__any_sync(0xffffffffu, move && j > 0)) {
      uint32_t orr[2][32];
      tmem_ld32(o_addr, orr[0]);
      tmem_ld32(o_addr + 32, orr[1]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) orr[c][e] = __float_as_uint(__uint_as_float(orr[c][e]) * alpha);
      tmem_st32(o_addr, orr[0]);
      tmem_st32(o_addr + 32, orr[1]);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar(BAR_P_FULL + tile));
  }
  // Merge the two halves of every row: both publish (m_h, l_h), then half h
  // writes output columns 32h .. 32h+31 from both accumulators.
  if (ok) {
    xchg[(tile * 2 + half) * BM + row] = make_float2(m_run, l_run);
    const uint32_t xbar = bar(BAR_XCHG + tile * 4 + quarter);
    mbar_arrive(xbar);
    ok = wait_bounded(xbar, 0, abort_flag, p.status, p.timeout_ns, 0x350u | tile) &&
         wait_bounded(bar(BAR_O_FINAL + tile), 0, abort_flag, p.status, p.timeout_ns, 0x320u | tile);
    ok = __all_sync(0xffffffffu, ok);
  }
  if (ok) {
    tc_fence_after();
    const float2 ml0 = xchg[(tile * 2 + 0) * BM + row];
    const float2 ml1 = xchg[(tile * 2 + 1) * BM + row];
    const float m = fmaxf(ml0.x, ml1.x);
    const float a0 = (ml0.x == -INFINITY) ? 0.f : ex2_approx(ml0.x - m);
    const float a1 = (ml1.x == -INFINITY) ? 0.f : ex2_approx(ml1.x - m);
    const float inv = 1.f / (a0 * ml0.y + a1 * ml1.y);
    const float w0 = a0 * inv, w1 = a1 * inv;
    uint32_t o0[32], o1[32];
    tmem_ld32(t_base + COL_O + half * 32, o0);        // O_i0, columns 32h..
    tmem_ld32(t_base + COL_O + D + half * 32, o1);    // O_i1, columns 32h..
    tmem_wait_ld();
    const int i = q0 + tile * BM + row;
    if (i < p.L) {
      const long long out_row = static_cast<long long>(b) * p.out_T +
                                static_cast<long long>(i / p.out_group) * p.out_T + (i % p.out_group);
      uint4* dst = reinterpret_cast<uint4*>(p.out + (out_row * p.H + h) * D + half * (D / 2));
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          f[e] = __uint_as_float(o0[v * 8 + e]) * w0 + __uint_as_float(o1[v * 8 + e]) * w1;
        uint4 w;
        w.x = pack_bf16x2(f[0], f[1]);
        w.y = pack_bf16x2(f[2], f[3]);
        w.z = pack_bf16x2(f[4], f[5]);
        w.w = pack_bf16x2(f[6], f[7]);
        dst[v] = w;
      }
    }
  }
}

__global__ void __launch_bounds__(core::THREADS, 1)
    attn_core_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const CoreParams p) {
  using namespace core;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float2* xchg = reinterpret_cast<float2*>(smem + OFF_XCHG);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = blockIdx.x * (NQ * BM);
  const int n_tiles = (q0 + BM < p.L) ? 2 : 1;          // the second Q tile may lie past the end
  const int n_kv = (p.L + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), n_tiles);   // one commit per MMA issuer
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_P_FULL + i), 256);
      mbar_init(bar(BAR_O_FINAL + i), 1);
    }
    for (int i = 0; i < NQ * 4; ++i) mbar_init(bar(BAR_XCHG + i), 64);
    for (int i = 0; i < NQ; ++i) mbar_init(bar(BAR_DRAIN + i), 1);
    fence_mbar_init();
    *abort_flag = status_is_set(p.status) ? 1 : 0;  // another CTA already failed: skip the work
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
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
    if (!skip && (((warp >> 2) - 1) >> 1) < n_tiles)
      softmax_role(p, tmem, bar0, xchg, abort_flag, h, b, q0, n_kv, warp, lane);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PRODUCER));
  }
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !skip) {
      int issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      mbar_arrive_expect_tx(bar(BAR_Q), n_tiles * TILE_BYTES);
      for (int i = 0; i < n_tiles; ++i)
        tma_load_3d(sbase + OFF_Q + i * TILE_BYTES, &tmap_q, bar(BAR_Q), 0, q0 + i * BM, b * p.H + h);
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % STAGES;
        if (j >= STAGES) {
          ok = wait_bounded(bar(BAR_KV_EMPTY + st), ((j / STAGES) - 1) & 1, abort_flag, p.status, p.timeout_ns,
                            0x100u | st);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bar(BAR_KV_FULL + st), 2 * TILE_BYTES);
        tma_load_3d(sbase + OFF_K + st * TILE_BYTES, &tmap_k, bar(BAR_KV_FULL + st), 0, j * BN, b * p.H + h);
        tma_load_4d(sbase + OFF_V + st * TILE_BYTES, &tmap_v, bar(BAR_KV_FULL + st), 0, h, j * BN, b);
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
    // Warp 1 issues every MMA of Q tile 0, warp 2 those of Q tile 1: one
    // thread can issue a tcgen05.mma only every ~45-50 cycles, so the two
    // tiles' instruction streams go out in parallel.  Within a tile the order
    // PV(j-1), S(j) is one thread's program order.
    const int i = warp - 1;
    if (lane == 0 && !skip && i < n_tiles) {
      // Descriptors differ only in their start-address field (address >> 4).
      const uint64_t dq = smem_desc_sw128(sbase + OFF_Q + i * TILE_BYTES, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sbase + OFF_K, 16, 1024);
      const uint64_t dv = smem_desc_sw128(sbase + OFF_V, 16384, 1024);
      const uint32_t t_tile = tmem + i * TILE_COLS;
      auto issue_s = [&](int st) {
        const uint64_t k = dk + st * (TILE_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(t_tile, dq + 2 * kk, k + 2 * kk, IDESC_QK, kk > 0);
      };
      // Key half hh: P at columns 64 hh .. of the tile's S (32 columns for 64
      // keys), V rows 64 hh .. of the stage, accumulator O_i,hh.
      auto issue_pv = [&](int st, bool acc) {
        const uint64_t v = dv + st * (TILE_BYTES >> 4);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int kk = 0; kk < HALF / 16; ++kk)
            mma_ts(t_tile + COL_O + hh * D, t_tile + hh * HALF + kk * 8, v + (hh * (HALF / 16) + kk) * (2048 >> 4),
                   IDESC_PV, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bounded(bar(BAR_Q), 0, abort_flag, p.status, p.timeout_ns, 0x200u) &&
                wait_bounded(bar(BAR_KV_FULL), 0, abort_flag, p.status, p.timeout_ns, 0x210u);
      // Stagger the two tiles by about half a period: tile 1 starts once tile
      // 0's first softmax is done, so the two softmax phases alternate.
      if (ok && i == 1) ok = wait_bounded(bar(BAR_P_FULL + 0), 0, abort_flag, p.status, p.timeout_ns, 0x2F0u);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        tc_commit(bar(BAR_S_FULL + i));
      }
      for (int j = 1; j < n_kv && ok; ++j) {
        const int st = j % STAGES, stp = (j - 1) % STAGES;
        ok = wait_bounded(bar(BAR_KV_FULL + st), (j / STAGES) & 1, abort_flag, p.status, p.timeout_ns,
                          0x210u | st) &&
             wait_bounded(bar(BAR_P_FULL + i), (j - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x220u | i);
        if (!ok) break;
        tc_fence_after();
        issue_pv(stp, j > 1);
        issue_s(st);
        tc_commit(bar(BAR_S_FULL + i));
        tc_commit(bar(BAR_KV_EMPTY + stp));
      }
      if (ok) {
        const int jl = n_kv - 1, stl = jl % STAGES;
        ok = wait_bounded(bar(BAR_P_FULL + i), jl & 1, abort_flag, p.status, p.timeout_ns, 0x230u | i);
        if (ok) {
          tc_fence_after();
          issue_pv(stl, jl > 0);
          tc_commit(bar(BAR_O_FINAL + i));
          tc_commit(bar(BAR_KV_EMPTY + stl));
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
