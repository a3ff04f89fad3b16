// Frame-mode attention core with persistent CTAs (VGGT-Omega Aggregator
// explainer, section 3, step 1: each frame's tokens attend within the frame).
//
// A frame problem has only ceil(T/80) = 13 key steps per 128-query tile, so a
// CTA that computes one tile spends a large share of its life starting up
// (barrier set-up, TMEM allocation, first loads from HBM) and draining.  Here
// each CTA (two per SM, 256 threads, 256 TMEM columns) walks the units
// u = blockIdx.x, blockIdx.x + gridDim.x, ... (unit = one 128-query tile of
// one (frame, head), tiles of a problem consecutive) and keeps its pipeline
// running across units: the producer loads the next unit's Q into the one Q
// buffer as soon as the current Q is in TMEM (a unit ahead of its use) and its
// K/V into the same ring, the softmax warps copy the next Q into TMEM as soon
// as the current unit's last QK^T product has completed, so the next unit's
// first products run during this unit's epilogue.  The epilogue writes the
// output tile through a shared-memory staging tile with one TMA store (rows
// past the frame's end are clipped by the tensor map); a thread's 128-byte
// output row would otherwise be a global store to a line of its own.  The
// per-step work is that of attn_core_kernel (see attention_sm100.cuh) -- Q in
// TMEM, two S buffers, online softmax with a lazily moved reference max --
// with two differences that fit the 256 TMEM columns of a CTA that shares its
// SM: steps of 80 keys (2 x 80 S + 64 O + 32 Q columns; 9 MMAs per 80 keys
// against 8 per 64, the per-instruction cost of these small products being
// what paces the loop), and row sums kept in registers by the softmax threads
// (fp32 sums of the probabilities before their rounding to bf16) instead of
// 16 ones columns in the PV product.  From its second step on, a tile's
// exponentials run against the reference max as it stands while the step's
// row max is taken in the same loop (ALU work beside the MUFU work, instead of
// a max pass ahead of them); in the rare step whose max exceeds the reference
// by more than the threshold they are redone against the new max, so P is the
// same as with the max taken first.  P goes into TMEM in three stores issued
// from inside the exponential loop as its parts are ready, so that the stores
// overlap the remaining exponentials.  Barrier phases run on across units.
// Every wait is bounded.
#pragma once

#include <cstdint>

#include "attention_sm100.cuh"

namespace vggt {

namespace fp {
using core::BM;
using core::D;
using core::Q_BYTES;
constexpr int BN = 80;                                  // keys per step
constexpr int KV_BYTES = BN * D * 2;                    // 10 KB key or value tile
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);   // V is MN-major
constexpr int STAGES = 4;
constexpr int OFF_Q = 0;                                // one Q buffer
constexpr int OFF_STG = OFF_Q + Q_BYTES;                // output staging tile (128 rows x 128 B)
constexpr int OFF_K = OFF_STG + Q_BYTES;
constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
constexpr int OFF_BAR = OFF_V + STAGES * KV_BYTES;
enum {
  BAR_Q_FULL = 0,
  BAR_Q_EMPTY = BAR_Q_FULL + 1,
  BAR_KV_FULL = BAR_Q_EMPTY + 1,
  BAR_KV_EMPTY = BAR_KV_FULL + STAGES,
  BAR_S_FULL = BAR_KV_EMPTY + STAGES,   // [buffer]
  BAR_P_FULL = BAR_S_FULL + 2,          // [buffer]
  BAR_PV_DONE = BAR_P_FULL + 2,
  BAR_O_FINAL = BAR_PV_DONE + 1,
  BAR_O_FREE = BAR_O_FINAL + 1,         // O read out by the epilogue
  BAR_Q_TMEM = BAR_O_FREE + 1,          // Q copied into TMEM
  BAR_DRAIN = BAR_Q_TMEM + 1,
  N_BARS = BAR_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;          // tmem slot, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES;   // base declared 1024-aligned; checked at entry
constexpr int THREADS = 256;
constexpr int CTAS_PER_SM = 2;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_O = 2 * BN;                      // S buffers at 0 and 80
constexpr uint32_t COL_Q = COL_O + D;
constexpr int REGS_AT_LAUNCH = 128;
constexpr int REGS_PRODUCER = 56;
constexpr int REGS_SOFTMAX = 200;
static_assert(REGS_PRODUCER * 128 + REGS_SOFTMAX * 128 <= REGS_AT_LAUNCH * THREADS, "register split too large");
// 228 KB of shared memory per SM, 1 KB of it reserved per resident CTA
static_assert((SMEM_ALLOC + 1024) * CTAS_PER_SM <= 228 * 1024, "two CTAs per SM");
static_assert(COL_Q + 32 <= TMEM_COLS, "TMEM layout");
}  // namespace fp

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

struct FrameUnits {
  int n_qt;       // 128-query tiles per (frame, head)
  int n_units;    // n_qt * H * S
};

__device__ __forceinline__ void frame_unit(const CoreParams& p, const FrameUnits& fu, int u, int& q0, int& h, int& b) {
  const int qt = u % fu.n_qt;
  const int r = u / fu.n_qt;
  h = r % p.H;
  b = r / p.H;
  q0 = qt * fp::BM;
}

__device__ __forceinline__ void mbar_arrive_count(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Softmax warpgroup (warps 4-7): thread r owns query row r of every unit.
__device__ __forceinline__ void frame_softmax_role(const CoreParams& p, const FrameUnits& fu, const uint8_t* smem,
                                                   const CUtensorMap& tmap_o, uint32_t tmem, uint32_t bar0,
                                                   volatile int* abort_flag, int n_kv, int warp, int lane) {
  using namespace fp;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t s_base = tmem + lane_base;
  const uint32_t o_addr = tmem + lane_base + COL_O;
  const PolyConsts pc = poly_consts();
  const bool leader = (threadIdx.x & 127) == 0;

  // Q tile of local unit i (128-byte swizzle) -> TMEM columns
  // COL_Q.. (row r in lane r, dims (2c, 2c+1) in column c).
  auto copy_q = [&](int i) -> bool {
    bool ok = wait_bounded(bar(BAR_Q_FULL), i & 1, abort_flag, p.status, p.timeout_ns, 0x630u);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    const uint4* qrow = reinterpret_cast<const uint4*>(smem + OFF_Q + row * 128);
    uint32_t qr[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 v = qrow[c ^ (row & 7)];
      qr[4 * c] = v.x;
      qr[4 * c + 1] = v.y;
      qr[4 * c + 2] = v.z;
      qr[4 * c + 3] = v.w;
    }
    tmem_st32(tmem + lane_base + COL_Q, qr);
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(bar(BAR_Q_TMEM));
    mbar_arrive(bar(BAR_Q_EMPTY));
    return true;
  };

  bool ok = true;
  bool q_ready = false;
  int G = 0;                                    // key steps done by this CTA
  const int c_pv = n_kv < 2 ? n_kv : 2;         // PV_DONE commits per unit
  for (int i = 0;; ++i) {
    const int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (u >= fu.n_units) break;
    int q0, h, b;
    frame_unit(p, fu, u, q0, h, b);
    if (!q_ready) {
      ok = copy_q(i);
      if (!ok) break;
    }
    q_ready = false;
    const int kv0 = i * n_kv;
    float m_run = -INFINITY;
    float l_run = 0.f;
    for (int j = 0; j < n_kv; ++j) {
      const int g = G + j;
      const int buf = g & 1;
      const uint32_t s_addr = s_base + buf * BN;
      ok = wait_bounded(bar(BAR_S_FULL + buf), (g >> 1) & 1, abort_flag, p.status, p.timeout_ns, 0x600u);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // S(j) complete => PV(j-2) complete: its K/V stage is free.
      if (j >= 2 && leader) mbar_arrive(bar(BAR_KV_EMPTY + (kv0 + j - 2) % STAGES));
      tc_fence_after();
      uint32_t sr[BN];
      tmem_ld32(s_addr, *reinterpret_cast<uint32_t(*)[32]>(sr));
      tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
      tmem_ld16(s_addr + 64, sr + 64);
      tmem_wait_ld();
      const int valid = p.Lk - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e >= valid) sr[e] = __float_as_uint(-INFINITY);
      }
      // Reference max for this step's exponentials: the running one, or on a
      // tile's first step this step's own max (taken first).
      float m_use = m_run;
      if (j == 0) {
        float a0 = -INFINITY, a1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < BN; e += 4) {
          a0 = max3f(a0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          a1 = max3f(a1, __uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3]));
        }
        m_use = fmaxf(a0, a1);
        m_run = m_use;
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
      float l0 = 0.f, l1 = 0.f;
      auto exps = [&](float neg_m, bool track) {
        uint32_t pk[BN / 2];
        l0 = 0.f;
        l1 = 0.f;
#pragma unroll
        for (int e = 0; e < BN; e += 2) {
          if (track) {
            if ((e & 2) == 0) mx0 = max3f(mx0, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
            else mx1 = max3f(mx1, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
          }
          float x0, x1, p0, p1;
          add_x2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), neg_m, neg_m, x0, x1);
          const int pair = e >> 1;
          if ((core::POLY_PAIR_MASK >> (pair & 7)) & 1u) {
            exp2_poly_x2(x0, x1, p0, p1, pc);
          } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          add_x2(l0, l1, p0, p1, l0, l1);
          pk[e >> 1] = pack_bf16x2(p0, p1);
          // P (80 keys -> 40 bf16-pair columns) over the first 40 columns of this S buffer, in parts as produced
          if (e == 30) tmem_st16(s_addr, pk);
          if (e == 62) tmem_st16(s_addr + 16, pk + 16);
          if (e == 78) tmem_st8(s_addr + 32, pk + 32);
        }
      };
      exps(-m_use, true);
      const float tile_max = fmaxf(mx0, mx1);
      const bool move = (j > 0) && (tile_max > m_run + core::RESCALE_THRESHOLD);
      float alpha = 1.f;
      if (move) {
        alpha = ex2_approx(m_run - tile_max);
        m_run = tile_max;
      }
      if (__any_sync(0xffffffffu, move)) {   // rare: P and its sum again against the moved max (warp-collective stores)
        tmem_wait_st();
        exps(-m_run, false);
      }
      // Row sum: this step's fp32 probabilities (two add chains) on top of
      // the running sum, which moves with the reference max as O does.
      l_run = l_run * alpha + (l0 + l1);
      // Rescale O after PV(j-1) (S(j+1) was issued after it; past the unit's
      // last S, the unit's first PV_DONE commit says so).
      if (__any_sync(0xffffffffu, move && j > 0)) {
        ok = (j + 1 < n_kv) ? wait_bounded(bar(BAR_S_FULL + ((g + 1) & 1)), ((g + 1) >> 1) & 1, abort_flag, p.status,
                                           p.timeout_ns, 0x610u)
                            : wait_bounded(bar(BAR_PV_DONE), (i * c_pv) & 1, abort_flag, p.status, p.timeout_ns,
                                           0x618u);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
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
      mbar_arrive(bar(BAR_P_FULL + buf));
    }
    if (!ok) break;
    // Next unit's Q into TMEM now (every QK^T product of this unit is done),
    // so that its first products run during this epilogue.
    if (u + static_cast<int>(gridDim.x) < fu.n_units) {
      ok = copy_q(i + 1);
      if (!ok) break;
      q_ready = true;
    }
    ok = wait_bounded(bar(BAR_O_FINAL), i & 1, abort_flag, p.status, p.timeout_ns, 0x620u);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    tc_fence_after();
    if (leader)
      for (int j = n_kv > 2 ? n_kv - 2 : 0; j < n_kv; ++j) mbar_arrive(bar(BAR_KV_EMPTY + (kv0 + j) % STAGES));
    uint32_t orr[2][32];
    tmem_ld32(o_addr, orr[0]);
    tmem_ld32(o_addr + 32, orr[1]);
    tmem_wait_ld();
    tc_fence_before();
    mbar_arrive(bar(BAR_O_FREE));
    // Output tile: each row into the staging tile (128-byte swizzle), then one
    // TMA store of the tile (rows past the frame's end are clipped by the map).
    {
      const bool issuer = (threadIdx.x & 127) == 0;
      if (issuer) bulk_wait_read_all();            // the previous unit's store has read the staging tile
      named_bar_sync(1, 128);
      const float inv = 1.f / l_run;
      uint4* srow = reinterpret_cast<uint4*>(const_cast<uint8_t*>(smem) + OFF_STG + row * 128);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 w;
          const uint32_t* o = &orr[c][v * 8];
          w.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
          srow[(c * 4 + v) ^ (row & 7)] = w;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      named_bar_sync(1, 128);
      if (issuer && VGGT_DBG_BOUNDS(h < p.H && q0 < p.L && b < p.B, p.status, 0x910u)) {
        tma_store_4d(&tmap_o, smem_addr(smem) + OFF_STG, 0, h, q0, b);
        bulk_commit();
      }
    }
    G += n_kv;
  }
  if ((threadIdx.x & 127) == 0) bulk_wait_all();
}

// Grid: min(n_units, 2 x SMs) CTAs, one dimension.  The producer runs ahead
// of the softmax by up to one unit of Q and STAGES key steps of K/V.
// tmap_o: out[S][T][H][64] as (dim, head, token, frame), box 64 x 1 x 128 x 1.
__global__ void __launch_bounds__(fp::THREADS, fp::CTAS_PER_SM)
    attn_frame_persistent_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                                 const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                                 const CoreParams p, const FrameUnits fu) {
  using namespace fp;
  using core::NV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if ((smem_addr(smem_raw) & 1023u) != 0) {   // the tiles need 1024-byte alignment and there is no slack
    if (threadIdx.x == 0) record_error(p.status, VGGT_ATTN_ERR_CUDA, 0x6F0u);
    return;
  }
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_kv = (p.Lk + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q_FULL), 1);
    mbar_init(bar(BAR_Q_EMPTY), 128);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), 1);
    }
    for (int buf = 0; buf < 2; ++buf) {
      mbar_init(bar(BAR_S_FULL + buf), 1);
      mbar_init(bar(BAR_P_FULL + buf), 128);
    }
    mbar_init(bar(BAR_PV_DONE), 1);
    mbar_init(bar(BAR_O_FINAL), 1);
    mbar_init(bar(BAR_O_FREE), 128);
    mbar_init(bar(BAR_Q_TMEM), 128);
    mbar_init(bar(BAR_DRAIN), 1);
    fence_mbar_init();
    *abort_flag = status_is_set(p.status) ? 1 : 0;  // another CTA already failed: skip the work
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
    tma_prefetch_desc(&tmap_o);
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
    if (!skip) frame_softmax_role(p, fu, smem, tmap_o, tmem, bar0, abort_flag, n_kv, warp, lane);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(REGS_PRODUCER));
  }
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && !skip) {
      int kv_issued[STAGES];
      for (int s = 0; s < STAGES; ++s) kv_issued[s] = 0;
      int q_issued = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
        if (u >= fu.n_units) break;
        int q0, h, b;
        frame_unit(p, fu, u, q0, h, b);
        if (i >= 1) {   // unit i-1's Q has been copied into TMEM
          ok = wait_bounded(bar(BAR_Q_EMPTY), (i - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x580u);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bar(BAR_Q_FULL), Q_BYTES);
        tma_load_3d(sbase + OFF_Q, &tmap_q, bar(BAR_Q_FULL), 0, q0, h * p.B + b);
        ++q_issued;
        for (int j = 0; j < n_kv; ++j) {
          const int k = i * n_kv + j;
          const int st = k % STAGES;
          if (k >= STAGES) {
            ok = wait_bounded(bar(BAR_KV_EMPTY + st), ((k / STAGES) - 1) & 1, abort_flag, p.status, p.timeout_ns,
                              0x500u | st);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(bar(BAR_KV_FULL + st), 2 * KV_BYTES);
          tma_load_3d(sbase + OFF_K + st * KV_BYTES, &tmap_k, bar(BAR_KV_FULL + st), 0, j * BN, h * p.B + b);
          tma_load_4d(sbase + OFF_V + st * KV_BYTES, &tmap_v, bar(BAR_KV_FULL + st), 0, h, j * BN, b);
          ++kv_issued[st];
        }
      }
      if (!ok) {
        // Drain: the last load issued into every stage and Q buffer must land
        // before this CTA's shared memory is released.
        if (q_issued > 0) wait_drain(bar(BAR_Q_FULL), (q_issued - 1) & 1, p.timeout_ns);
        for (int st = 0; st < STAGES; ++st)
          if (kv_issued[st] > 0) wait_drain(bar(BAR_KV_FULL + st), (kv_issued[st] - 1) & 1, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip) {
      const uint64_t dk = smem_desc_sw128(sbase + OFF_K, 16, 1024);
      const uint32_t t_o = tmem + COL_O, t_q = tmem + COL_Q;
      auto issue_s = [&](int g, int k) {   // S of step g into buffer g % 2, K from load k, Q from TMEM
        const uint64_t kd = dk + (k % STAGES) * (KV_BYTES >> 4);
        const uint32_t d = tmem + (g & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ts(d, t_q + kk * 8, kd + 2 * kk, IDESC_QK, kk > 0);
      };
      auto issue_pv = [&](int g, int k, bool first) {   // O (+)= P(g) [V(k) | 1]
        const uint32_t v_addr = sbase + OFF_V + (k % STAGES) * KV_BYTES;
        const uint64_t v = smem_desc_sw128(v_addr, KV_BYTES, 1024);   // N = 64: one swizzle atom wide
        const uint32_t a = tmem + (g & 1) * BN;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(t_o, a + kk * 8, v + kk * (2048 >> 4), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
      };
      bool ok = true;
      int G = 0;
      for (int i = 0; ok; ++i) {
        const int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
        if (u >= fu.n_units) break;
        const int kv0 = i * n_kv;
        ok = wait_bounded(bar(BAR_Q_TMEM), i & 1, abort_flag, p.status, p.timeout_ns, 0x540u);
        for (int jj = 0; jj < 2 && jj < n_kv && ok; ++jj) {
          const int k = kv0 + jj;
          ok = wait_bounded(bar(BAR_KV_FULL + k % STAGES), (k / STAGES) & 1, abort_flag, p.status, p.timeout_ns,
                            0x510u | jj);
          if (!ok) break;
          tc_fence_after();
          issue_s(G + jj, k);
          tc_commit(bar(BAR_S_FULL + ((G + jj) & 1)));
        }
        for (int j = 0; j < n_kv && ok; ++j) {
          const int g = G + j;
          const int jn = j + 2;
          if (jn < n_kv) {   // K/V of step j+2 first (normally long resident)
            const int kn = kv0 + jn;
            ok = wait_bounded(bar(BAR_KV_FULL + kn % STAGES), (kn / STAGES) & 1, abort_flag, p.status,
                              p.timeout_ns, 0x530u);
            if (!ok) break;
          }
          ok = wait_bounded(bar(BAR_P_FULL + (g & 1)), (g >> 1) & 1, abort_flag, p.status, p.timeout_ns, 0x520u);
          if (!ok) break;
          if (j == 0 && i > 0) {   // the previous unit's epilogue has read O
            ok = wait_bounded(bar(BAR_O_FREE), (i - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x550u);
            if (!ok) break;
          }
          tc_fence_after();
          issue_pv(g, kv0 + j, j == 0);
          if (jn < n_kv) {
            issue_s(g + 2, kv0 + jn);
            tc_commit(bar(BAR_S_FULL + (g & 1)));   // also covers PV(j)
          } else {
            tc_commit(bar(BAR_PV_DONE));
            if (j == n_kv - 1) tc_commit(bar(BAR_O_FINAL));
          }
        }
        G += n_kv;
      }
      if (!ok) {  // let every MMA already issued finish before TMEM is released
        tc_commit(bar(BAR_DRAIN));
        wait_drain(bar(BAR_DRAIN), 0, p.timeout_ns);
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

}  // namespace vggt
