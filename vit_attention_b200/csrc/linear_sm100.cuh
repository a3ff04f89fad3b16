// Dense projections either side of the attention core on sm_100a (tcgen05 +
// TMEM + TMA): Y = X W^T + b with X [M][K], W [N][K] (nn.Linear weight
// layout), bf16 operands and fp32 accumulation.
// (VGGT-Omega Aggregator explainer, section 3: every attention block of the
// alternating-attention layer projects its 1024 channels to q, k, v and its
// attention output back to 1024 channels.)
//
// Two epilogues:
//   plain  -- bf16(Y) into y[M][N] (the output projection, or an unfused qkv);
//   qkv    -- the QKV projection of a frame or global attention block: the
//             columns of a 64-wide head slice of q or k go through the QK
//             LayerNorm, the 2D RoPE and (q) the softmax scale in fp32 straight
//             from the accumulator and land in the attention workspace in the
//             core's layout [B][H][L][64]; v slices go to the v slot of
//             qkv[S][T][3][H][64].  This replaces the separate prologue pass
//             and its HBM round trip of q and k.
//
// Persistent CTAs (one per SM) walk 128 x 256 output tiles (n fastest).  Warp
// roles (256 threads):
//   warp 0       TMA producer: X tile 128 x 64 and W tile 256 x 64 per k-step
//                (128-byte swizzle, no multicast) into a 4-stage ring.
//   warp 1       MMA issuer (and TMEM owner): 4 x tcgen05.mma M=128 N=256 K=16
//                per k-step into one of two 256-column TMEM accumulators, so
//                the epilogue of one tile overlaps the products of the next.
//   warps 4-7    epilogue: thread r owns output row r of the tile (TMEM lane r);
//                it reads 64 accumulator columns at a time, adds the bias and
//                stores bf16 (or normalises/rotates, in the qkv epilogue).
// Every mbarrier wait is bounded (wait_bounded); on expiry the CTA records
// VGGT_ATTN_ERR_TIMEOUT in the status word and drains what it has in flight.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

namespace lin {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;                   // 16 KB
constexpr int B_BYTES = BN * BK * 2;                   // 32 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_BAR = OFF_B + STAGES * B_BYTES;
enum {
  BAR_FULL = 0,
  BAR_EMPTY = BAR_FULL + STAGES,
  BAR_ACC_FULL = BAR_EMPTY + STAGES,   // [accumulator]
  BAR_ACC_EMPTY = BAR_ACC_FULL + 2,    // [accumulator]
  BAR_DRAIN = BAR_ACC_EMPTY + 2,
  N_BARS = BAR_DRAIN + 1
};
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;         // tmem slot, abort flag
constexpr int OFF_ROPE = OFF_MISC + 16;                // cos/sin table (qkv epilogue)
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;                    // two 256-column accumulators
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 0);
constexpr int REGS_AT_LAUNCH = 168;
}  // namespace lin

struct LinearParams {
  int M, N, K;
  const float* bias;          // [N] or null
  uint16_t* y;                // plain epilogue: [M][N]
  int* status;
  unsigned long long timeout_ns;
  int zero_status;            // clear the status word first (the first kernel of an attention block)
  // qkv epilogue (fused == 1); N = 3 * H * 64, K = H * 64
  int fused;
  uint16_t* ws_qk[2];         // q, k destinations [B][H][L][64]
  uint16_t* qkv;              // v destination: qkv[M][3][H][64]
  const float* gamma[2];
  const float* beta[2];
  int H, T, L, n_special, grid_h, grid_w;
  float eps, q_mult, rope_base;
};

__host__ __device__ inline int linear_smem_bytes(int grid_h, int grid_w) {
  return lin::OFF_ROPE + (grid_h + grid_w) * 16 * 8 + 1024;   // + slack to align the base to 1024 B
}

// 32 lanes x 64 columns load.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// Epilogue of one 128 x 256 tile: thread `row` owns output row m0 + row; acc
// is its TMEM lane at the tile's accumulator.
__device__ __forceinline__ void linear_epilogue(const LinearParams& p, uint32_t acc, int m0, int n0, int row,
                                                const float2* rope_tab) {
  const int m = m0 + row;
  const bool valid = m < p.M;
#pragma unroll 1
  for (int ck = 0; ck < lin::BN / 64; ++ck) {
    uint32_t r[64];
    tmem_ld64(acc + ck * 64, r);
    tmem_wait_ld();
    const int col0 = n0 + ck * 64;
    float x[64];
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
      const float4 bv = p.bias ? __ldg(reinterpret_cast<const float4*>(p.bias + col0 + e)) : make_float4(0.f, 0.f, 0.f, 0.f);
      x[e] = __uint_as_float(r[e]) + bv.x;
      x[e + 1] = __uint_as_float(r[e + 1]) + bv.y;
      x[e + 2] = __uint_as_float(r[e + 2]) + bv.z;
      x[e + 3] = __uint_as_float(r[e + 3]) + bv.w;
    }
    const int c = p.fused ? col0 / (p.H * 64) : 2;   // 0 q, 1 k, 2 v (or plain)
    if (!valid) continue;
    if (c == 2) {
      uint16_t* dst = (p.fused ? p.qkv : p.y) + static_cast<size_t>(m) * p.N + col0;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * v], x[8 * v + 1]);
        w.y = pack_bf16x2(x[8 * v + 2], x[8 * v + 3]);
        w.z = pack_bf16x2(x[8 * v + 4], x[8 * v + 5]);
        w.w = pack_bf16x2(x[8 * v + 6], x[8 * v + 7]);
        reinterpret_cast<uint4*>(dst)[v] = w;
      }
      continue;
    }
    // QK LayerNorm over the head's 64 values (biased variance, two passes).
    const int h = (col0 / 64) % p.H;
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 64; ++e) sum += x[e];
    const float mean = sum * (1.0f / 64.0f);
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      x[e] -= mean;
      sq += x[e] * x[e];
    }
    const float rstd = rsqrtf(sq * (1.0f / 64.0f) + p.eps);
    const float* gm = p.gamma[c] + h * 64;
    const float* bt = p.beta[c] + h * 64;
#pragma unroll
    for (int e = 0; e < 64; e += 4) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(gm + e));
      const float4 b4 = __ldg(reinterpret_cast<const float4*>(bt + e));
      x[e] = x[e] * rstd * g4.x + b4.x;
      x[e + 1] = x[e + 1] * rstd * g4.y + b4.y;
      x[e + 2] = x[e + 2] * rstd * g4.z + b4.z;
      x[e + 3] = x[e + 3] * rstd * g4.w + b4.w;
    }
    // 2D RoPE on patch tokens: dims [0,32) by row, [32,64) by column, pairs (j, j+16).
    const int t = m % p.T;
    if (t >= p.n_special) {
      const int pp = t - p.n_special;
      const int prow = pp / p.grid_w, pcol = pp - prow * p.grid_w;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float2* cs = rope_tab + (half == 0 ? prow : p.grid_h + pcol) * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float2 v = cs[j];
          const float a = x[32 * half + j], b = x[32 * half + j + 16];
          x[32 * half + j] = a * v.x - b * v.y;
          x[32 * half + j + 16] = b * v.x + a * v.y;
        }
      }
    }
    const float mult = (c == 0) ? p.q_mult : 1.0f;
    const int b = m / p.L, pos = m - b * p.L;
    uint16_t* dst = p.ws_qk[c] + ((static_cast<size_t>(b) * p.H + h) * p.L + pos) * 64;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      uint4 w;
      w.x = pack_bf16x2(x[8 * v] * mult, x[8 * v + 1] * mult);
      w.y = pack_bf16x2(x[8 * v + 2] * mult, x[8 * v + 3] * mult);
      w.z = pack_bf16x2(x[8 * v + 4] * mult, x[8 * v + 5] * mult);
      w.w = pack_bf16x2(x[8 * v + 6] * mult, x[8 * v + 7] * mult);
      reinterpret_cast<uint4*>(dst)[v] = w;
    }
  }
}

__global__ void __launch_bounds__(lin::THREADS, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const LinearParams p) {
  using namespace lin;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float2* rope_tab = reinterpret_cast<float2*>(smem + OFF_ROPE);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM, tiles_n = p.N / BN, n_tiles = tiles_m * tiles_n;
  const int k_steps = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(BAR_FULL + s), 1);
      mbar_init(bar(BAR_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(BAR_ACC_FULL + a), 1);
      mbar_init(bar(BAR_ACC_EMPTY + a), 128);
    }
    mbar_init(bar(BAR_DRAIN), 1);
    fence_mbar_init();
    *abort_flag = 0;
    if (p.zero_status && blockIdx.x == 0) {
      p.status[0] = 0;
      p.status[1] = 0;
    }
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (p.fused) {
    const int n_pos = p.grid_h + p.grid_w;
    for (int e = threadIdx.x; e < n_pos * 16; e += blockDim.x) {
      const int pos_idx = e >> 4, j = e & 15;
      const double pos = pos_idx < p.grid_h ? pos_idx : pos_idx - p.grid_h;
      const double omega = pow(static_cast<double>(p.rope_base), -static_cast<double>(j) / 16.0);
      double s, c;
      sincos(pos * omega, &s, &c);
      rope_tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
    }
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
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int st = it % STAGES;
          if (it >= STAGES) {
            ok = wait_bounded(bar(BAR_EMPTY + st), ((it / STAGES) - 1) & 1, abort_flag, p.status, p.timeout_ns,
                              0x500u | st);
            if (!ok) break;
          }
          mbar_arrive_expect_tx(bar(BAR_FULL + st), A_BYTES + B_BYTES);
          tma_load_3d(sbase + OFF_A + st * A_BYTES, &tmap_x, bar(BAR_FULL + st), k * BK, m0, 0);
          tma_load_3d(sbase + OFF_B + st * B_BYTES, &tmap_w, bar(BAR_FULL + st), k * BK, n0, 0);
          ++issued[st];
        }
      }
      if (!ok) {
        for (int st = 0; st < STAGES; ++st)
          if (issued[st] > 0) wait_drain(bar(BAR_FULL + st), (issued[st] - 1) & 1, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !skip) {
      const uint64_t da = smem_desc_sw128(sbase + OFF_A, 16, 1024);
      const uint64_t db = smem_desc_sw128(sbase + OFF_B, 16, 1024);
      bool ok = true;
      int it = 0, lt = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        if (lt >= 2) {
          ok = wait_bounded(bar(BAR_ACC_EMPTY + ab), ((lt >> 1) - 1) & 1, abort_flag, p.status, p.timeout_ns,
                            0x510u | ab);
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t d = tmem + ab * BN;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int st = it % STAGES;
          ok = wait_bounded(bar(BAR_FULL + st), (it / STAGES) & 1, abort_flag, p.status, p.timeout_ns, 0x520u | st);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(d, da + st * (A_BYTES >> 4) + 2 * kk, db + st * (B_BYTES >> 4) + 2 * kk, IDESC,
                   (k > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(BAR_EMPTY + st));
        }
        if (ok) tc_commit(bar(BAR_ACC_FULL + ab));
      }
      if (!ok) {
        tc_commit(bar(BAR_DRAIN));
        wait_drain(bar(BAR_DRAIN), 0, p.timeout_ns);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    if (!skip) {
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      int lt = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        bool ok = wait_bounded(bar(BAR_ACC_FULL + ab), (lt >> 1) & 1, abort_flag, p.status, p.timeout_ns,
                               0x530u | ab);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        linear_epilogue(p, tmem + lane_base + ab * BN, m0, n0, row, rope_tab);
        tc_fence_before();
        mbar_arrive(bar(BAR_ACC_EMPTY + ab));
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
