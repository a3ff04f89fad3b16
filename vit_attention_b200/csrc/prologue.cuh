// QK-LayerNorm + 2D RoPE prologue (VGGT-Omega Aggregator explainer,
// section 3: "use_qk_norm=True" and the 2D RoPE re-applied at every layer).
//
// Reads the q and k rows of the packed bf16 qkv[S][T][3][H][64], normalises
// each 64-dim head vector (biased variance, per-head affine), rotates patch
// tokens, multiplies q by softmax_scale*log2(e) (so the core works in base 2)
// and writes bf16 into the workspace in the attention core's layout
//   q, k : [B][H][L][64]   (frame: B = S, L = T; global: B = 1, L = S*T;
//                           register: B = 1, L = S*n_special)
//   v    : [L][H][64]      (register mode only: the gathered special tokens)
//
// HBM-bound: 8 threads own one 128-byte head row (16 bytes each); the 8-lane
// groups of a block cover the n_c*H contiguous head rows of a token, and each
// lane keeps four tokens' loads in flight.  The LayerNorm reductions are 3
// shuffles inside the 8-lane group, and a RoPE pair (j, j+16) sits in lanes g
// and g^2 of the group.  The cos/sin table of every (row|col position,
// frequency) is built once per block in fp64 and kept in shared memory as
// fp32.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

struct PrologueParams {
  const uint16_t* qkv;
  const float* gamma[2];  // q, k
  const float* beta[2];
  uint16_t* ws_qk[2];     // q, k destinations
  uint16_t* ws_v;         // register mode only
  int* status;
  long long n_rows;       // n_tok * n_c * H
  int S, T, H, n_special, grid_h, grid_w;
  int mode;               // VGGT_ATTN_FRAME / GLOBAL / REGISTER
  int L;                  // tokens per problem in the workspace
  int n_c;                // 2 (q, k) or 3 (q, k, v in register mode)
  float eps;
  float q_mult;           // softmax_scale * log2(e)
  float rope_base;
};

// Where one 128-byte head row (token i of the mode's token list, tensor c,
// head h) lives and goes.
struct PrologueRow {
  int c, h, t;                 // q/k/v, head, token inside its frame
  long long src;               // element offset of the row in qkv
  long long dst;               // element offset in the destination buffer
};

__device__ __forceinline__ PrologueRow prologue_row(const PrologueParams& p, int i, int c, int h) {
  PrologueRow w;
  w.c = c;
  w.h = h;
  int flat, b, pos;                              // token index into S*T; problem, position in the workspace
  if (p.mode == VGGT_ATTN_REGISTER) {
    const int s = i / p.n_special;
    flat = s * p.T + (i - s * p.n_special);
    b = 0;
    pos = i;
  } else {
    flat = i;
    b = i / p.L;
    pos = i - b * p.L;
  }
  w.t = flat - (flat / p.T) * p.T;
  w.src = ((static_cast<long long>(flat) * 3 + c) * p.H + h) * 64;
  w.dst = (c == 2) ? (static_cast<long long>(pos) * p.H + h) * 64
                   : ((static_cast<long long>(b) * p.H + h) * p.L + pos) * 64;
  return w;
}

// LayerNorm + RoPE (+ q scale) of the 8 values this lane holds of one row,
// written back as bf16.  Every lane of the 8-lane group calls it together.
__device__ __forceinline__ void prologue_finish(const PrologueParams& p, const PrologueRow& w, uint4 raw, int g,
                                                unsigned gmask, const float2* rope_tab) {
  if (w.c == 2) {  // register-mode v gather: plain copy
    *reinterpret_cast<uint4*>(p.ws_v + w.dst + g * 8) = raw;
    return;
  }
  float x[8];
  const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    x[2 * e] = __uint_as_float(wd[e] << 16);
    x[2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
  }
  // LayerNorm over the 64 values held by the 8-lane group (two passes).
  float sum = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) sum += x[e];
  sum += __shfl_xor_sync(gmask, sum, 1);
  sum += __shfl_xor_sync(gmask, sum, 2);
  sum += __shfl_xor_sync(gmask, sum, 4);
  const float mean = sum * (1.0f / 64.0f);
  float sq = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    x[e] -= mean;
    sq += x[e] * x[e];
  }
  sq += __shfl_xor_sync(gmask, sq, 1);
  sq += __shfl_xor_sync(gmask, sq, 2);
  sq += __shfl_xor_sync(gmask, sq, 4);
  const float rstd = rsqrtf(sq * (1.0f / 64.0f) + p.eps);
  const float4* gm = reinterpret_cast<const float4*>(p.gamma[w.c] + w.h * 64 + g * 8);
  const float4* bt = reinterpret_cast<const float4*>(p.beta[w.c] + w.h * 64 + g * 8);
  const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1), b0 = __ldg(bt), b1 = __ldg(bt + 1);
  const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) x[e] = x[e] * rstd * gg[e] + bb[e];

  // 2D RoPE on patch tokens.  Lanes 0-3 hold dims 0-31 (row), 4-7 dims
  // 32-63 (col); lanes with bit 1 clear hold the first member j of a pair
  // (j, j+16), their partner is lane g^2.  The branch is uniform over the
  // 8-lane group, the shuffles run in every lane of the group.
  const bool is_patch = w.t >= p.n_special;
  float partner[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) partner[e] = __shfl_xor_sync(gmask, x[e], 2);
  if (is_patch) {
    const int pp = w.t - p.n_special;
    const int prow = pp / p.grid_w, pcol = pp - prow * p.grid_w;
    const int pos_idx = (g < 4) ? prow : p.grid_h + pcol;
    const int j0 = 8 * (g & 1);
    const bool second = (g & 2) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 cs = rope_tab[pos_idx * 16 + j0 + e];
      x[e] = second ? (x[e] * cs.x + partner[e] * cs.y) : (x[e] * cs.x - partner[e] * cs.y);
    }
  }
  if (w.c == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= p.q_mult;
  }
  uint4 o;
  o.x = pack_bf16x2(x[0], x[1]);
  o.y = pack_bf16x2(x[2], x[3]);
  o.z = pack_bf16x2(x[4], x[5]);
  o.w = pack_bf16x2(x[6], x[7]);
  *reinterpret_cast<uint4*>(p.ws_qk[w.c] + w.dst + g * 8) = o;
}

__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const PrologueParams p) {
  extern __shared__ float2 rope_tab[];  // [(grid_h + grid_w) * 16]: (cos, sin)
  const int n_pos = p.grid_h + p.grid_w;
  for (int e = threadIdx.x; e < n_pos * 16; e += blockDim.x) {
    const int pos_idx = e >> 4, j = e & 15;
    const double pos = pos_idx < p.grid_h ? pos_idx : pos_idx - p.grid_h;
    const double omega = pow(static_cast<double>(p.rope_base), -static_cast<double>(j) / 16.0);
    double s, c;
    sincos(pos * omega, &s, &c);
    rope_tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.status[0] = 0;
    p.status[1] = 0;
  }
  __syncthreads();

  const int g = threadIdx.x & 7;                    // lane inside the 8-lane row group
  // Shuffles involve only the 8 lanes of one row group: the groups of a warp
  // may take different paths (v rows, loop tail).
  const unsigned gmask = 0xFFu << (threadIdx.x & 24);
  // Block iteration: TOKENS tokens (blockIdx.x + k * gridDim.x); the block's
  // 8-lane groups cover the n_c * H head rows of a token, which are contiguous
  // in qkv (n_c*H*128 bytes), so every load instruction of the block reads
  // whole lines and TOKENS loads are in flight per lane.
  constexpr int TOKENS = 4;
  const int n_tok = static_cast<int>(p.n_rows / (p.n_c * p.H));   // < 2^31 (checked on the host)
  const int ch = p.n_c * p.H;
  const int groups = blockDim.x >> 3, gi = threadIdx.x >> 3;
  for (int i0 = blockIdx.x; i0 < n_tok; i0 += TOKENS * gridDim.x) {
    for (int idx = gi; idx < ch; idx += groups) {     // uniform over the 8-lane group
      const int c = idx / p.H, h = idx - c * p.H;
      PrologueRow w[TOKENS];
      uint4 raw[TOKENS];
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        const int ik = i0 + k * gridDim.x;
        w[k] = prologue_row(p, ik < n_tok ? ik : i0, c, h);
      }
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) raw[k] = *reinterpret_cast<const uint4*>(p.qkv + w[k].src + g * 8);
#pragma unroll
      for (int k = 0; k < TOKENS; ++k)
        if (i0 + k * gridDim.x < n_tok) prologue_finish(p, w[k], raw[k], g, gmask, rope_tab);
    }
  }
}

}  // namespace vggt
