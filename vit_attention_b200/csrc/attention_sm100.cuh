// Exact softmax attention core for head_dim 64 on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA computes one 128-query tile of one (problem, head):
//   O = softmax(Q K^T) V   over the problem's L keys, Q already scaled by
//   softmax_scale*log2(e) (the prologue does it), so scores are in base 2.
// (VGGT-Omega Aggregator explainer, section 3: the frame / global / register
// attention of the alternating-attention block; the kernel is the same for
// the three modes, only the workspace views and the output row map differ.)
//
// Warp roles (192 threads):
//   warp 0      TMA producer: the Q tile once, then K/V tiles of 128 keys
//               through a 4-stage shared-memory ring (128-byte swizzle).
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma:
//               S[j%2] = Q K_j^T   (M=128, N=128, K=16 x 4)  -> TMEM, fp32
//               O     += P_j V_j   (M=128, N=64,  K=16 x 8)  P read from TMEM
//   warps 2..5  softmax: thread r owns query row r (= TMEM lane r); reads its
//               128 scores from TMEM, keeps a running max m and sum l in fp32,
//               writes P = 2^(s - m) as bf16 back over the S columns, and
//               rescales O in TMEM when m grows by more than 8 (= a factor of
//               256; below that the stale max is kept, which is exact because
//               O and l always share the same m).  Epilogue: O / l -> bf16.
//
// TMEM (512 columns): S/P buffer 0 at col 0, buffer 1 at col 128, O at col 256.
// Every mbarrier wait is bounded (wait_bounded); on expiry the CTA records
// VGGT_ATTN_ERR_TIMEOUT in the workspace status word, drains what it has in
// flight and exits without writing its output tile.
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
constexpr int BM = 128, BN = 128, D = 64, STAGES = 4;
constexpr int TILE_BYTES = BM * D * 2;                 // 16 KB (Q, K or V tile)
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_V = OFF_K + STAGES * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + STAGES * TILE_BYTES;  // 147456
enum {
  BAR_Q = 0,
  BAR_KV_FULL = 1,
  BAR_KV_EMPTY = BAR_KV_FULL + STAGES,
  BAR_S_FULL = BAR_KV_EMPTY + STAGES,
  BAR_P_FULL = BAR_S_FULL + 2,
  BAR_PV_DONE = BAR_P_FULL + 2,
  BAR_O_FINAL = BAR_PV_DONE + 1,
  BAR_DRAIN = BAR_O_FINAL + 1,
  N_BARS = BAR_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;         // tmem slot, abort flag
constexpr int SMEM_BYTES = OFF_MISC + 16;
constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;          // slack to align the base to 1024 B
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t COL_O = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;              // log2 units
constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);  // V is MN-major (head dim contiguous)
}  // namespace core

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
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int q0 = qt * BM;
  const int n_kv = (p.L + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(bar(BAR_Q), 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_S_FULL + i), 1);
      mbar_init(bar(BAR_P_FULL + i), 128);
    }
    mbar_init(bar(BAR_PV_DONE), 1);
    mbar_init(bar(BAR_O_FINAL), 1);
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
      int issued[STAGES] = {0, 0, 0, 0};
      mbar_arrive_expect_tx(bar(BAR_Q), TILE_BYTES);
      tma_load_3d(sbase + OFF_Q, &tmap_q, bar(BAR_Q), 0, q0, b * p.H + h);
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
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
      bool ok = wait_bounded(bar(BAR_Q), 0, abort_flag, p.status, p.timeout_ns, 0x200u);
      const uint32_t q_addr = sbase + OFF_Q;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j % STAGES, sb = j & 1;
        ok = wait_bounded(bar(BAR_KV_FULL + st), (j / STAGES) & 1, abort_flag, p.status, p.timeout_ns,
                          0x210u | st);
        if (!ok) break;
        if (j >= 2) {  // S/P buffer sb is free once PV(j-2) has completed
          ok = wait_bounded(bar(BAR_PV_DONE), (j - 2) & 1, abort_flag, p.status, p.timeout_ns, 0x220u);
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t k_addr = sbase + OFF_K + st * TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ss(tmem + sb * BN, smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                 smem_desc_sw128(k_addr + kk * 32, 16, 1024), IDESC_QK, kk > 0);
        }
        tc_commit(bar(BAR_S_FULL + sb));
        if (j >= 1) {
          const int jp = j - 1, stp = jp % STAGES, sbp = jp & 1;
          ok = wait_bounded(bar(BAR_P_FULL + sbp), (jp >> 1) & 1, abort_flag, p.status, p.timeout_ns, 0x230u);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_addr = sbase + OFF_V + stp * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            mma_ts(tmem + COL_O, tmem + sbp * BN + kk * 8, smem_desc_sw128(v_addr + kk * 2048, 16384, 1024),
                   IDESC_PV, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(BAR_KV_EMPTY + stp));
          tc_commit(bar(BAR_PV_DONE));
        }
      }
      if (ok) {
        const int jp = n_kv - 1, stp = jp % STAGES, sbp = jp & 1;
        ok = wait_bounded(bar(BAR_P_FULL + sbp), (jp >> 1) & 1, abort_flag, p.status, p.timeout_ns, 0x240u);
        if (ok) {
          tc_fence_after();
          const uint32_t v_addr = sbase + OFF_V + stp * TILE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            mma_ts(tmem + COL_O, tmem + sbp * BN + kk * 8, smem_desc_sw128(v_addr + kk * 2048, 16384, 1024),
                   IDESC_PV, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar(BAR_KV_EMPTY + stp));
          tc_commit(bar(BAR_O_FINAL));
        }
      }
      if (!ok) {  // let every MMA already issued finish before TMEM is released
        tc_commit(bar(BAR_DRAIN));
        wait_drain(bar(BAR_DRAIN), 0, p.timeout_ns);
      }
    }
  } else if (!skip) {
    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3;              // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;       // query row of this thread in the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      ok = wait_bounded(bar(BAR_S_FULL + sb), (j >> 1) & 1, abort_flag, p.status, p.timeout_ns, 0x300u);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_base + sb * BN;
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
      tmem_wait_ld();
      const int valid = p.L - j * BN;          // keys of this tile that exist (may be < 128 on the last)
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float s = __uint_as_float(sr[c][e]);
          if (c * 32 + e >= valid) s = -INFINITY;
          sr[c][e] = __float_as_uint(s);
          mx = fmaxf(mx, s);
        }
      }
      // Conditional rescale: move the reference max only when it grows by
      // more than the threshold (always on the first tile).
      const bool move = (j == 0) || (mx > m_run + RESCALE_THRESHOLD);
      float alpha = 1.f;
      if (move) {
        alpha = (j == 0) ? 0.f : ex2_approx(m_run - mx);
        m_run = mx;
      }
      float lsum = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float p0 = ex2_approx(__uint_as_float(sr[c][e]) - m_run);
          const float p1 = ex2_approx(__uint_as_float(sr[c][e + 1]) - m_run);
          lsum += p0 + p1;
          pk[c >> 1][(c & 1) * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
        }
      }
      // P overwrites the first 64 columns of this S buffer (2 bf16 per column).
      tmem_st32(s_addr, pk[0]);
      tmem_st32(s_addr + 32, pk[1]);
      l_run = l_run * alpha + lsum;
      // O must be rescaled before PV(j) accumulates into it; PV(j-1) has to be
      // finished first.  Warp-uniform: tcgen05.ld/st are warp-collective.
      const bool need = __any_sync(0xffffffffu, move && j > 0);
      if (need) {
        ok = wait_bounded(bar(BAR_PV_DONE), (j - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x310u);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t o_addr = tmem + lane_base + COL_O;
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
      mbar_arrive(bar(BAR_P_FULL + sb));
    }
    if (ok) {
      ok = wait_bounded(bar(BAR_O_FINAL), 0, abort_flag, p.status, p.timeout_ns, 0x320u);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      uint32_t orr[2][32];
      tmem_ld32(tmem + lane_base + COL_O, orr[0]);
      tmem_ld32(tmem + lane_base + COL_O + 32, orr[1]);
      tmem_wait_ld();
      const int i = q0 + row;
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
