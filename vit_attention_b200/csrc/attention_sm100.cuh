// Exact softmax attention core for head_dim 64 on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA computes two 128-query tiles (256 queries) of one (problem, head):
//   O = softmax(Q K^T) V   over the problem's L keys.  Q arrives scaled by
//   softmax_scale*log2(e) from the prologue, so scores are in base 2.
// (VGGT-Omega Aggregator explainer, section 3: the frame / global / register
// attention of the alternating-attention block; the kernel is the same for
// the three modes, only the workspace views and the output row map differ.)
//
// Warp roles (384 threads, 12 warps):
//   warp 0       TMA producer: both Q tiles once, then K/V tiles of 128 keys
//                through a shared-memory ring (128-byte swizzle, no multicast).
//   warp 1       TMEM allocator; lane 0 issues every tcgen05.mma:
//                  S_i = Q_i K_j^T (M=128, N=128, K=16 x 4, fp32 in TMEM)
//                  O_i += P_i V_j  (M=128, N=64,  K=16 x 8, P read from TMEM)
//                in the order PV_0(j-1), S_0(j), PV_1(j-1), S_1(j), so the
//                tensor core works on one tile while the other tile's softmax
//                runs, and the commit that publishes S_i(j) also proves that
//                PV_i(j-1) has finished.
//   warps 2-3    idle.
//   warps 4-7    softmax of tile 0, warps 8-11 softmax of tile 1: thread r of
//                a warpgroup owns query row r (= TMEM lane r).  Per key tile it
//                reads its 128 scores from TMEM, keeps a running max m and sum
//                l in fp32, writes P = 2^(s - m) as bf16 over the first 64 S
//                columns, and rescales O_i in TMEM only when m grows by more
//                than 8 (a factor of 256; below that the stale max is kept,
//                which is exact because O and l always share the same m).
//                Part of the exponentials run on the FMA pipe (a cubic for
//                2^f after an exponent split), the rest on the MUFU unit.
//                Epilogue: O / l -> bf16 -> out.
//
// TMEM (512 columns allocated): S/P_0 at col 0, S/P_1 at col 128, O_0 at col
// 256, O_1 at col 320.  Every mbarrier wait is bounded (wait_bounded); on
// expiry the CTA records VGGT_ATTN_ERR_TIMEOUT in the workspace status word,
// drains what it has in flight and exits without writing its output tiles.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

struct CoreParams {
  int L;              // keys (and queries) per problem
  int H;              // heads
  int out_T;          // tokens per frame of `out`
  int out_group;      // query i of problem b -> out row b*out_T + (i/out_group)*out_T + i%out_group
  uint16_t* out;      // bf16 [.][H][64]
  int* status;
  unsigned long long timeout_ns;
};

namespace core {
constexpr int BM = 128, BN = 128, D = 64, STAGES = 4, NQ = 2;
constexpr int TILE_BYTES = BM * D * 2;                 // 16 KB (Q, K or V tile)
constexpr int OFF_Q = 0;                               // NQ tiles
constexpr int OFF_K = OFF_Q + NQ * TILE_BYTES;
constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;
enum {
  BAR_Q = 0,
  BAR_KV_FULL = 1,
  BAR_KV_EMPTY = BAR_KV_FULL + STAGES,
  BAR_S_FULL = BAR_KV_EMPTY + STAGES,
  BAR_P_FULL = BAR_S_FULL + NQ,
  BAR_O_FINAL = BAR_P_FULL + NQ,
  BAR_DRAIN = BAR_O_FINAL + NQ,
  N_BARS = BAR_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;         // tmem slot, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;          // slack to align the base to 1024 B
constexpr int THREADS = 384;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;              // log2 units
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);  // V is MN-major (head dim contiguous)
// Exponentials of score pair q (0..63 in a row) run on the FMA pipe when
// bit (q % 8) of this mask is set (3 of 8 pairs), on the MUFU unit otherwise.
constexpr uint32_t POLY_PAIR_MASK = 0x92u;
}  // namespace core

// 2^x for x <= ~128 on the FMA pipe, two values at once: x = j + f with
// j = round(x) (via the 1.5*2^23 shift), f in [-1/2, 1/2]; 2^f from a cubic
// fitted by minimax in relative error (fit_exp2_poly.py, max rel. error
// 7.5e-5); 2^j added to the exponent field.  x is clamped at -125 so that the
// exponent field never underflows (2^-125 is far below any probability that
// survives bf16 rounding next to the row maximum's 1).
__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& y0, float& y1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  float t0, t1, r0, r1, f0, f1, p0, p1;
  asm("{\n\t.reg .b64 rx, rs, rt, rr, rf, rp, rc;\n\t"
      "mov.b64 rx, {%8, %9};\n\t"
      "mov.b64 rs, {%10, %10};\n\t"
      "add.rn.f32x2 rt, rx, rs;\n\t"          // t = x + shift (integer part in the low mantissa)
      "sub.rn.f32x2 rr, rt, rs;\n\t"          // r = round(x)
      "sub.rn.f32x2 rf, rx, rr;\n\t"          // f = x - r
      "mov.b64 rc, {%11, %11};\n\t"
      "mov.b64 rp, {%12, %12};\n\t"
      "fma.rn.f32x2 rp, rc, rf, rp;\n\t"      // c3 f + c2
      "mov.b64 rc, {%13, %13};\n\t"
      "fma.rn.f32x2 rp, rp, rf, rc;\n\t"      // (..) f + c1
      "mov.b64 rc, {%14, %14};\n\t"
      "fma.rn.f32x2 rp, rp, rf, rc;\n\t"      // (..) f + c0
      "mov.b64 {%0, %1}, rt;\n\t"
      "mov.b64 {%2, %3}, rr;\n\t"
      "mov.b64 {%4, %5}, rf;\n\t"
      "mov.b64 {%6, %7}, rp;\n\t}"
      : "=f"(t0), "=f"(t1), "=f"(r0), "=f"(r1), "=f"(f0), "=f"(f1), "=f"(p0), "=f"(p1)
      : "f"(x0), "f"(x1), "f"(kShift), "f"(5.517166853e-02f), "f"(2.426111251e-01f), "f"(6.932609677e-01f),
        "f"(9.999280572e-01f));
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z;
  const int q0 = blockIdx.x * (NQ * BM);
  const int n_tiles = (q0 + BM < p.L) ? 2 : 1;          // the second Q tile may lie past the end
  const int n_kv = (p.L + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), 1);
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_P_FULL + i), 128);
      mbar_init(bar(BAR_O_FINAL + i), 1);
    }
    mbar_init(bar(BAR_DRAIN), 1);
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip) {
      auto issue_s = [&](int i, int st) {
        const uint32_t q_addr = sbase + OFF_Q + i * TILE_BYTES;
        const uint32_t k_addr = sbase + OFF_K + st * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + i * BN, smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                 smem_desc_sw128(k_addr + kk * 32, 16, 1024), IDESC_QK, kk > 0);
      };
      auto issue_pv = [&](int i, int st, bool acc) {
        const uint32_t v_addr = sbase + OFF_V + st * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          mma_ts(tmem + COL_O + i * D, tmem + i * BN + kk * 8, smem_desc_sw128(v_addr + kk * 2048, 16384, 1024),
                 IDESC_PV, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bounded(bar(BAR_Q), 0, abort_flag, p.status, p.timeout_ns, 0x200u) &&
                wait_bounded(bar(BAR_KV_FULL), 0, abort_flag, p.status, p.timeout_ns, 0x210u);
      if (ok) {
        tc_fence_after();
        for (int i = 0; i < n_tiles; ++i) {
          issue_s(i, 0);
          tc_commit(bar(BAR_S_FULL + i));
        }
      }
      for (int j = 1; j < n_kv && ok; ++j) {
        const int st = j % STAGES, stp = (j - 1) % STAGES;
        ok = wait_bounded(bar(BAR_KV_FULL + st), (j / STAGES) & 1, abort_flag, p.status, p.timeout_ns,
                          0x210u | st);
        for (int i = 0; i < n_tiles && ok; ++i) {
          ok = wait_bounded(bar(BAR_P_FULL + i), (j - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x220u | i);
          if (!ok) break;
          tc_fence_after();
          issue_pv(i, stp, j > 1);
          issue_s(i, st);
          tc_commit(bar(BAR_S_FULL + i));
        }
        if (ok) tc_commit(bar(BAR_KV_EMPTY + stp));
      }
      if (ok) {
        const int jl = n_kv - 1, stl = jl % STAGES;
        for (int i = 0; i < n_tiles && ok; ++i) {
          ok = wait_bounded(bar(BAR_P_FULL + i), jl & 1, abort_flag, p.status, p.timeout_ns, 0x230u | i);
          if (!ok) break;
          tc_fence_after();
          issue_pv(i, stl, jl > 0);
          tc_commit(bar(BAR_O_FINAL + i));
        }
        if (ok) tc_commit(bar(BAR_KV_EMPTY + stl));
      }
      if (!ok) {  // let every MMA already issued finish before TMEM is released
        tc_commit(bar(BAR_DRAIN));
        wait_drain(bar(BAR_DRAIN), 0, p.timeout_ns);
      }
    }
  } else if (warp >= 4 && !skip && ((warp >> 2) - 1) < n_tiles) {
    // ------------------------------------------------------------ softmax warpgroups
    const int tile = (warp >> 2) - 1;
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;       // query row of this thread in its tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + tile * BN;
    const uint32_t o_addr = tmem + lane_base + COL_O + tile * D;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = wait_bounded(bar(BAR_S_FULL + tile), j & 1, abort_flag, p.status, p.timeout_ns, 0x300u | tile);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
      tmem_wait_ld();
      const int valid = p.L - j * BN;          // keys of this tile that exist
      if (valid < BN) {                        // last tile only (uniform branch)
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e >= valid) sr[c][e] = __float_as_uint(-INFINITY);
      }
      float mx[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float a = __uint_as_float(sr[c][0]), bb = __uint_as_float(sr[c][1]);
#pragma unroll
        for (int e = 2; e < 32; e += 2) {
          a = max3f(a, __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
        }
        mx[c] = fmaxf(a, bb);
      }
      const float tile_max = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // Conditional rescale: move the reference max only when it grows by
      // more than the threshold (always on the first tile).
      const bool move = (j == 0) || (tile_max > m_run + RESCALE_THRESHOLD);
      float alpha = 1.f;
      if (move) {
        alpha = (j == 0) ? 0.f : ex2_approx(m_run - tile_max);
        m_run = tile_max;
      }
      const float neg_m = -m_run;
      float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = half * 2 + cc;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float x0, x1, p0, p1;
            add_x2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]), neg_m, neg_m, x0, x1);
            const int pair = (c * 32 + e) >> 1;
            if ((POLY_PAIR_MASK >> (pair & 7)) & 1u) {
              exp2_poly_x2(x0, x1, p0, p1);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
            }
            if (e & 2) {
              add_x2(acc2, acc3, p0, p1, acc2, acc3);
            } else {
              add_x2(acc0, acc1, p0, p1, acc0, acc1);
            }
            pk[cc * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
          }
        }
        // P overwrites the first 64 columns of this tile's S (2 bf16 per column).
        tmem_st32(s_addr + half * 32, pk);
      }
      l_run = l_run * alpha + ((acc0 + acc1) + (acc2 + acc3));
      // O_i must be rescaled before PV_i(j) accumulates into it.  PV_i(j-1)
      // is complete: the commit that published S_i(j) came after it.
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
    if (ok) {
      ok = wait_bounded(bar(BAR_O_FINAL + tile), 0, abort_flag, p.status, p.timeout_ns, 0x320u | tile);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      uint32_t orr[2][32];
      tmem_ld32(o_addr, orr[0]);
      tmem_ld32(o_addr + 32, orr[1]);
      tmem_wait_ld();
      const int i = q0 + tile * BM + row;
      if (i < p.L) {
        const float inv = 1.f / l_run;
        const long long out_row = static_cast<long long>(b) * p.out_T +
                                  static_cast<long long>(i / p.out_group) * p.out_T + (i % p.out_group);
        uint4* dst = reinterpret_cast<uint4*>(p.out + (out_row * p.H + h) * D);
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
            dst[c * 4 + v] = w;
          }
        }
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
