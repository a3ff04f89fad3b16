// Dense projections either side of the attention core on sm_100a (tcgen05 +
// TMEM + TMA): Y = X W^T + b with X [M][K], W [N][K] (nn.Linear weight
// layout), bf16 operands and fp32 accumulation.
// (VGGT-Omega Aggregator explainer, section 3: every attention block of the
// alternating-attention layer projects its 1024 channels to q, k, v and its
// attention output back to 1024 channels.)
//
// Epilogues (the template argument EPI picks one; each is its own kernel):
//   plain  -- bf16(Y) into y[M][N] (the output projection, or an unfused qkv);
//   gelu   -- bf16(GELU(Y)) into y (the MLP's first layer; exact erf form);
//   resid  -- y = r + ls * Y with r a bf16 [M][N] residual and ls a per-column
//             LayerScale vector, into y (may be r itself: each element is read
//             by the thread that then writes it, before the chunk's store);
//   qkv    -- (EPI_QKV) the QKV projection of a frame or global attention block: the
//             columns of a 64-wide head slice of q or k go through the QK
//             LayerNorm, the 2D RoPE and (q) the softmax scale in fp32 straight
//             from the accumulator and land in the attention workspace in the
//             core's layout (one [S*T][64] plane per head); v slices go to the
//             v slot of qkv[S][T][3][H][64].  This replaces the separate
//             prologue pass and its HBM round trip of q and k.
// Every 64-column chunk of a tile is staged in shared memory (128-byte
// swizzle) and written by one TMA store: whole lines, rows past M clipped.
//
// Persistent CTAs (one per SM) walk 128 x 256 output tiles (n fastest).  Warp
// roles (256 threads):
//   warp 0       TMA producer: X tile 128 x 64 and W tile 256 x 64 per k-step
//                (128-byte swizzle, no multicast) into a 4-stage ring.
//   warp 1       MMA issuer (and TMEM owner): 4 x tcgen05.mma M=128 N=256 K=16
//                per k-step into one of two 256-column TMEM accumulators, so
//                the epilogue of one tile overlaps the products of the next.
//   warps 4-7    epilogue: thread r owns output row r of the tile (TMEM lane r);
//                it reads 64 accumulator columns at a time, adds the bias,
//                (qkv epilogue: normalises and rotates), and writes its 128-byte
//                row of the chunk into the staging buffer; one thread stores
//                the chunk with TMA.
//   warps 8-11   (gelu, resid and qkv epilogues, 384 threads) a second
//                epilogue warpgroup: warps 4-7 take chunks 0-1 of every tile,
//                warps 8-11 chunks 2-3, each with its own staging buffer, so
//                that the heavier per-element work keeps up with the products
//                (5 % off a frame-mode transformer block for gelu/resid).  The
//                qkv epilogue also keeps its cos/sin table in shared memory, so
//                its operand ring has 3 stages instead of 4 to make room.
// Every mbarrier wait is bounded (wait_bounded); on expiry the CTA records
// VGGT_ATTN_ERR_TIMEOUT in the status word and drains what it has in flight.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

namespace lin {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
enum { EPI_STD = 0, EPI_GELU = 1, EPI_RESID = 2, EPI_QKV = 3 };
constexpr int A_BYTES = BM * BK * 2;                   // 16 KB
constexpr int B_BYTES = BN * BK * 2;                   // 32 KB
// Operand ring stages: 4, or 3 for the qkv epilogue (its cos/sin table and a
// second staging buffer take the fourth stage's shared memory).
__host__ __device__ constexpr int stages_for(int epi) { return epi == EPI_QKV ? 3 : STAGES; }
constexpr int OFF_A = 0;
__host__ __device__ constexpr int off_b(int epi) { return OFF_A + stages_for(epi) * A_BYTES; }
__host__ __device__ constexpr int off_stage(int epi) { return off_b(epi) + stages_for(epi) * B_BYTES; }  // 128 x 64 bf16 chunk
__host__ __device__ constexpr int off_bar(int epi) { return off_stage(epi) + BM * 128; }
enum {
  BAR_FULL = 0,
  BAR_EMPTY = BAR_FULL + STAGES,
  BAR_ACC_FULL = BAR_EMPTY + STAGES,   // [accumulator]
  BAR_ACC_EMPTY = BAR_ACC_FULL + 2,    // [accumulator]
  BAR_STAGE_FULL = BAR_ACC_EMPTY + 2,  // every epilogue thread wrote its row of the chunk
  BAR_STAGE_FREE = BAR_STAGE_FULL + 1, // the chunk's TMA store has read the buffer
  BAR_STAGE_FULL2 = BAR_STAGE_FREE + 1, // the same for the second epilogue warpgroup's buffer
  BAR_STAGE_FREE2 = BAR_STAGE_FULL2 + 1,
  BAR_DRAIN = BAR_STAGE_FREE2 + 1,
  N_BARS = BAR_DRAIN + 1
};
__host__ __device__ constexpr int off_misc(int epi) { return off_bar(epi) + N_BARS * 8; }   // tmem slot, abort flag
__host__ __device__ constexpr int off_rope(int epi) { return off_misc(epi) + 16; }          // cos/sin table (qkv)
constexpr int THREADS = 256;
// The GELU, residual and qkv epilogues do more per element: they run on two
// warpgroups (warps 4-7 take the tile's first two 64-column chunks, warps
// 8-11 the last two), each with its own staging buffer; the second buffer
// follows the cos/sin table of (grid_h + grid_w) positions (none but qkv).
__host__ __device__ constexpr int rope_bytes(int epi, int n_pos) { return epi == EPI_QKV ? n_pos * 16 * 8 : 0; }
__host__ __device__ constexpr int off_stage2(int epi, int n_pos) { return (off_rope(epi) + rope_bytes(epi, n_pos) + 1023) & ~1023; }
__host__ __device__ constexpr int epi_warpgroups(int epi) { return epi == EPI_STD ? 1 : 2; }
__host__ __device__ constexpr int threads_for(int epi) { return 128 * (1 + epi_warpgroups(epi)); }
constexpr uint32_t TMEM_COLS = 512;                    // two 256-column accumulators
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, 0);
constexpr int REGS_AT_LAUNCH = 168;
}  // namespace lin

struct LinearParams {
  int M, N, K;
  const float* bias;          // [N] or null
  int* status;
  unsigned long long timeout_ns;
  int zero_status;            // clear the status word first (the first kernel of an attention block)
  // qkv epilogue (EPI_QKV); N = 3 * H * 64, K = H * 64; the destinations
  // are the kernel's output tensor maps (v slot of qkv, q plane, k plane)
  const float* gamma[2];
  const float* beta[2];
  int H, T, n_special, grid_h, grid_w;
  float eps, q_mult, rope_base;
  // residual epilogue: y = resid + ls * (X W^T + b), resid bf16 [M][N]
  const uint16_t* resid;
  const float* ls;             // [N]
};

// + 1 KB of slack to align the base to 1024 B
__host__ __device__ constexpr int linear_smem_bytes(int grid_h, int grid_w, int epi = lin::EPI_STD) {
  if (epi != lin::EPI_STD) return lin::off_stage2(epi, grid_h + grid_w) + lin::BM * 128 + 1024;
  return lin::off_rope(epi) + 1024;
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

// Epilogue of one 128 x 256 tile: thread `row` owns output row m0 + row (its
// TMEM lane at the tile's accumulator is `acc`).  Each 64-column chunk is
// converted in registers, staged in shared memory and stored by the leader
// thread with one TMA store; `chunk` counts the CTA's chunks (barrier phases).
// Loads of bias, gamma and beta are issued a few at a time, so that the
// chunk's 64 values are the only large live state.
template <int EPI>
__device__ __forceinline__ bool linear_epilogue(const LinearParams& p, uint32_t acc, int m0, int n0, int row,
                                                bool leader, uint8_t* stage, uint32_t bar0, volatile int* abort_flag,
                                                int& chunk, const CUtensorMap* to0, const CUtensorMap* to1,
                                                const CUtensorMap* to2, const float2* rope_tab, int ck_begin,
                                                int ck_end, int bar_full, int bar_free) {
  using namespace lin;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int m = m0 + row;                 // rows past M compute garbage that TMA clips
  // Residual epilogue: the residual of the next chunk is loaded while this
  // one is converted (rows past M have none).
  uint4 rnext[8];
  if constexpr (EPI == lin::EPI_RESID) {
    const uint4* rrow = reinterpret_cast<const uint4*>(p.resid + static_cast<long long>(m) * p.N + n0 + ck_begin * 64);
#pragma unroll
    for (int k = 0; k < 8; ++k) rnext[k] = m < p.M ? rrow[k] : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll 1
  for (int ck = ck_begin; ck < ck_end; ++ck, ++chunk) {
    uint4 rcur[8];
    if constexpr (EPI == lin::EPI_RESID) {
#pragma unroll
      for (int k = 0; k < 8; ++k) rcur[k] = rnext[k];
      if (ck + 1 < ck_end) {
        const uint4* rrow = reinterpret_cast<const uint4*>(p.resid + static_cast<long long>(m) * p.N + n0 + (ck + 1) * 64);
#pragma unroll
        for (int k = 0; k < 8; ++k) rnext[k] = m < p.M ? rrow[k] : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    uint32_t v[64];
    tmem_ld64(acc + ck * 64, v);
    tmem_wait_ld();
    const int col0 = n0 + ck * 64;
    if (p.bias) {
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        const float4 bv = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + e));
        v[e] = __float_as_uint(__uint_as_float(v[e]) + bv.x);
        v[e + 1] = __float_as_uint(__uint_as_float(v[e + 1]) + bv.y);
        v[e + 2] = __float_as_uint(__uint_as_float(v[e + 2]) + bv.z);
        v[e + 3] = __float_as_uint(__uint_as_float(v[e + 3]) + bv.w);
      }
    }
    if constexpr (EPI == lin::EPI_GELU) {
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float x = __uint_as_float(v[e]);
        v[e] = __float_as_uint(0.5f * x * (1.0f + erff(x * 0.70710678118654752f)));   // x * Phi(x)
      }
    }
    if constexpr (EPI == lin::EPI_RESID) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint4 r = rcur[k];
        const float4 l0 = __ldg(reinterpret_cast<const float4*>(p.ls + col0 + 8 * k));
        const float4 l1 = __ldg(reinterpret_cast<const float4*>(p.ls + col0 + 8 * k + 4));
        const uint32_t rw[4] = {r.x, r.y, r.z, r.w};
        const float lv[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float r0 = __uint_as_float(rw[i] << 16), r1 = __uint_as_float(rw[i] & 0xFFFF0000u);
          v[8 * k + 2 * i] = __float_as_uint(r0 + lv[2 * i] * __uint_as_float(v[8 * k + 2 * i]));
          v[8 * k + 2 * i + 1] = __float_as_uint(r1 + lv[2 * i + 1] * __uint_as_float(v[8 * k + 2 * i + 1]));
        }
      }
    }
    const int c = EPI == lin::EPI_QKV ? col0 / (p.H * 64) : 2;   // 0 q, 1 k, 2 v (or plain)
    const int h = EPI == lin::EPI_QKV ? (col0 / 64) % p.H : 0;
    uint4 o[8];
    if (c == 2) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        o[k].x = pack_bf16x2(__uint_as_float(v[8 * k]), __uint_as_float(v[8 * k + 1]));
        o[k].y = pack_bf16x2(__uint_as_float(v[8 * k + 2]), __uint_as_float(v[8 * k + 3]));
        o[k].z = pack_bf16x2(__uint_as_float(v[8 * k + 4]), __uint_as_float(v[8 * k + 5]));
        o[k].w = pack_bf16x2(__uint_as_float(v[8 * k + 6]), __uint_as_float(v[8 * k + 7]));
      }
    } else if constexpr (EPI == lin::EPI_QKV) {
      // QK LayerNorm over the head's 64 values (biased variance, two passes;
      // eight partial sums each, then a short tree).
      float ps[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) ps[q] = __uint_as_float(v[q]);
#pragma unroll
      for (int e = 8; e < 64; ++e) ps[e & 7] += __uint_as_float(v[e]);
      const float mean = (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]))) * (1.0f / 64.0f);
#pragma unroll
      for (int q = 0; q < 8; ++q) ps[q] = 0.f;
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        const float d = __uint_as_float(v[e]) - mean;
        v[e] = __float_as_uint(d);
        ps[e & 7] += d * d;
      }
      const float sq = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      const float rstd = rsqrtf(sq * (1.0f / 64.0f) + p.eps);
      const float mult = (c == 0) ? p.q_mult : 1.0f;
      // Affine, then 2D RoPE on patch tokens (dims [0,32) by row, [32,64) by
      // column, pairs (j, j+16)), then the q scale; one 32-dim half at a time.
      const int t = m % p.T;
      const bool patch = t >= p.n_special;
      int prow = 0, pcol = 0;
      if (patch) {
        const int pp = t - p.n_special;
        prow = pp / p.grid_w;
        pcol = pp - prow * p.grid_w;
      }
      const float* gm = p.gamma[c] + h * 64;
      const float* bt = p.beta[c] + h * 64;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float2* cs = rope_tab + (hf == 0 ? prow : p.grid_h + pcol) * 16;
        // Dims d0..d0+3 and their RoPE partners d1 = d0 + 16: packed straight
        // into the output words (o[4 hf + j/8] holds dims 32 hf + j/8*8 ..,
        // o[4 hf + 2 + j/8] the partners).
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const int d0 = 32 * hf + j, d1 = d0 + 16;
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(gm + d0));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(gm + d1));
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(bt + d0));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(bt + d1));
          const float ga[4] = {g0.x, g0.y, g0.z, g0.w}, gb[4] = {g1.x, g1.y, g1.z, g1.w};
          const float ba[4] = {b0.x, b0.y, b0.z, b0.w}, bb[4] = {b1.x, b1.y, b1.z, b1.w};
          float ya[4], yb[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float a = __uint_as_float(v[d0 + i]) * rstd * ga[i] + ba[i];
            float bv = __uint_as_float(v[d1 + i]) * rstd * gb[i] + bb[i];
            if (patch) {
              const float2 w = cs[j + i];
              const float a2 = a * w.x - bv * w.y;
              bv = bv * w.x + a * w.y;
              a = a2;
            }
            ya[i] = a * mult;
            yb[i] = bv * mult;
          }
          uint4& oa = o[4 * hf + j / 8];
          uint4& ob = o[4 * hf + 2 + j / 8];
          if ((j & 4) == 0) {
            oa.x = pack_bf16x2(ya[0], ya[1]);
            oa.y = pack_bf16x2(ya[2], ya[3]);
            ob.x = pack_bf16x2(yb[0], yb[1]);
            ob.y = pack_bf16x2(yb[2], yb[3]);
          } else {
            oa.z = pack_bf16x2(ya[0], ya[1]);
            oa.w = pack_bf16x2(ya[2], ya[3]);
            ob.z = pack_bf16x2(yb[0], yb[1]);
            ob.w = pack_bf16x2(yb[2], yb[3]);
          }
        }
      }
    }
    // Stage the chunk: wait until the previous chunk's store has read the buffer.
    if (chunk > 0) {
      if (leader) {
        bulk_wait_read_all();
        mbar_arrive(bar(bar_free));
      }
      bool ok = wait_bounded(bar(bar_free), (chunk - 1) & 1, abort_flag, p.status, p.timeout_ns, 0x540u);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(stage + row * 128 + ((k ^ (row & 7)) * 16)) = o[k];
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive(bar(bar_full));
    bool ok = true;
    if (leader) {
      ok = wait_bounded(bar(bar_full), chunk & 1, abort_flag, p.status, p.timeout_ns, 0x550u);
      if (ok) {
        const uint32_t src = smem_addr(stage);
        if (EPI != lin::EPI_QKV)
          tma_store_3d(to0, src, col0, m0, 0);          // y [M][N]
        else if (c == 2)
          tma_store_4d(to0, src, 0, h, 2, m0);          // v slot of qkv [M][3][H][64]
        else
          tma_store_3d(c == 0 ? to1 : to2, src, 0, m0, h);   // q or k plane of head h
        bulk_commit();
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
  }
  return true;
}

template <int EPI>
__global__ void __launch_bounds__(lin::threads_for(EPI), 1)
    linear_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const __grid_constant__ CUtensorMap tmap_o0, const __grid_constant__ CUtensorMap tmap_o1,
                  const __grid_constant__ CUtensorMap tmap_o2, const LinearParams p) {
  using namespace lin;
  constexpr int NST = stages_for(EPI);
  constexpr int OFF_B = off_b(EPI), OFF_STAGE = off_stage(EPI), OFF_BAR = off_bar(EPI), OFF_MISC = off_misc(EPI);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const uint32_t bar0 = sbase + OFF_BAR;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float2* rope_tab = reinterpret_cast<float2*>(smem + off_rope(EPI));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_m = (p.M + BM - 1) / BM, tiles_n = p.N / BN, n_tiles = tiles_m * tiles_n;
  const int k_steps = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar(BAR_FULL + s), 1);
      mbar_init(bar(BAR_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(BAR_ACC_FULL + a), 1);
      mbar_init(bar(BAR_ACC_EMPTY + a), 128 * epi_warpgroups(EPI));
    }
    mbar_init(bar(BAR_STAGE_FULL), 128);
    mbar_init(bar(BAR_STAGE_FREE), 1);
    mbar_init(bar(BAR_STAGE_FULL2), 128);
    mbar_init(bar(BAR_STAGE_FREE2), 1);
    mbar_init(bar(BAR_DRAIN), 1);
    fence_mbar_init();
    *abort_flag = 0;
    if (p.zero_status && blockIdx.x == 0) {
      p.status[0] = 0;
      p.status[1] = 0;
    }
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    tma_prefetch_desc(&tmap_o0);
    if (EPI == EPI_QKV) {
      tma_prefetch_desc(&tmap_o1);
      tma_prefetch_desc(&tmap_o2);
    }
  }
  if (EPI == EPI_QKV) {
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
      int issued[NST];
      for (int s = 0; s < NST; ++s) issued[s] = 0;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int st = it % NST;
          if (it >= NST) {
            ok = wait_bounded(bar(BAR_EMPTY + st), ((it / NST) - 1) & 1, abort_flag, p.status, p.timeout_ns,
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
        for (int st = 0; st < NST; ++st)
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
          const int st = it % NST;
          ok = wait_bounded(bar(BAR_FULL + st), (it / NST) & 1, abort_flag, p.status, p.timeout_ns, 0x520u | st);
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
      const int wg = (warp - 4) >> 2;                        // epilogue warpgroup
      constexpr int CPW = (BN / 64) / epi_warpgroups(EPI);   // chunks per warpgroup
      const bool leader = (threadIdx.x & 127) == 0;
      uint8_t* stage = smem + (wg == 0 ? OFF_STAGE : off_stage2(EPI, p.grid_h + p.grid_w));
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      int lt = 0, chunk = 0;
      for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++lt) {
        const int ab = lt & 1;
        bool ok = wait_bounded(bar(BAR_ACC_FULL + ab), (lt >> 1) & 1, abort_flag, p.status, p.timeout_ns,
                               0x530u | ab);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int m0 = (t / tiles_n) * BM, n0 = (t % tiles_n) * BN;
        ok = linear_epilogue<EPI>(p, tmem + lane_base + ab * BN, m0, n0, row, leader, stage, bar0, abort_flag, chunk,
                                  &tmap_o0, &tmap_o1, &tmap_o2, rope_tab, wg * CPW, (wg + 1) * CPW,
                                  wg == 0 ? BAR_STAGE_FULL : BAR_STAGE_FULL2,
                                  wg == 0 ? BAR_STAGE_FREE : BAR_STAGE_FREE2);
        tc_fence_before();
        mbar_arrive(bar(BAR_ACC_EMPTY + ab));
        if (!ok) break;
      }
      if (leader) bulk_wait_all();   // the last stores have completed before the CTA exits
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
