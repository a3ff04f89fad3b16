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
// HBM-bound: 8 threads own one 128-byte head row (16 bytes each).  A block
// has one 8-lane group per head row of a token (n_c*H groups, n_c*H*128
// contiguous bytes of qkv), so a group keeps the same (tensor, head) for all
// the tokens it visits and holds that row's gamma/beta in registers; each
// lane keeps four tokens' loads in flight.  The LayerNorm reductions are 3
// shuffles inside the 8-lane group, and a RoPE pair (j, j+16) sits in lanes g
// and g^2 of the group.  Token -> (problem, position, frame slot) divisions
// use a multiply-high by a precomputed reciprocal with one correction step.
// The cos/sin table of every (row|col position, frequency) is built once per
// block in fp64 and kept in shared memory as fp32.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

// n / d and n % d for 0 <= n < 2^31 and d >= 1: m = ceil(2^32 / d) (2^32 - 1
// for d = 1), q = mulhi(n, m) is floor(n/d) or one more.
struct FastDiv {
  uint32_t d, m;
};
inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.m = d <= 1 ? 0xFFFFFFFFu : static_cast<uint32_t>(((1ull << 32) + d - 1) / d);
  return f;
}
__device__ __forceinline__ uint32_t fast_divmod(uint32_t n, const FastDiv& f, uint32_t& r) {
  uint32_t q = __umulhi(n, f.m);
  int rr = static_cast<int>(n - q * f.d);
  if (rr < 0) {
    --q;
    rr += static_cast<int>(f.d);
  } else if (rr >= static_cast<int>(f.d)) {
    ++q;
    rr -= static_cast<int>(f.d);
  }
  r = static_cast<uint32_t>(rr);
  return q;
}

struct PrologueParams {
  const uint16_t* qkv;
  const float* gamma[2];  // q, k
  const float* beta[2];
  uint16_t* ws_qk[2];     // q, k destinations
  uint16_t* ws_v;         // register mode only
  int* status;
  int n_tok;              // tokens in the mode's token list (< 2^31, checked on the host)
  int T, H, n_special, grid_h, grid_w;
  int mode;               // VGGT_ATTN_FRAME / GLOBAL / REGISTER
  int L;                  // tokens per problem in the workspace
  int n_c;                // 2 (q, k) or 3 (q, k, v in register mode)
  FastDiv div_nspec, div_L, div_T, div_gw;
  float eps;
  float q_mult;           // softmax_scale * log2(e)
  float rope_base;
};

// Where token i of the mode's token list comes from and goes to.
struct PrologueToken {
  long long src;          // element offset of the token's [3][H][64] block in qkv
  long long dst_qk;       // element offset of (problem, head 0, position) in q/k
  long long dst_v;        // element offset of (position, head 0) in the gathered v
  int t;                  // token index inside its frame
};

__device__ __forceinline__ PrologueToken prologue_token(const PrologueParams& p, uint32_t i) {
  uint32_t flat, b, pos;   // token index into S*T; problem, position in the workspace
  if (p.mode == VGGT_ATTN_REGISTER) {
    uint32_t r;
    const uint32_t s = fast_divmod(i, p.div_nspec, r);
    flat = s * static_cast<uint32_t>(p.T) + r;
    b = 0;
    pos = i;
  } else {
    flat = i;
    b = fast_divmod(i, p.div_L, pos);
  }
  PrologueToken w;
  uint32_t t;
  fast_divmod(flat, p.div_T, t);
  w.t = static_cast<int>(t);
  w.src = static_cast<long long>(flat) * 3 * p.H * 64;
  w.dst_qk = (static_cast<long long>(b) * p.H * p.L + pos) * 64;
  w.dst_v = static_cast<long long>(pos) * p.H * 64;
  return w;
}

__global__ void __launch_bounds__(384) qk_norm_rope_kernel(const PrologueParams p) {
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
  constexpr int TOKENS = 4;
  const int ch = p.n_c * p.H;
  const int groups = blockDim.x >> 3;
  for (int idx = threadIdx.x >> 3; idx < ch; idx += groups) {   // uniform over the 8-lane group
    const int c = idx / p.H, h = idx - c * p.H;
    float gg[8], bb[8];
    if (c < 2) {
      const float4* gm = reinterpret_cast<const float4*>(p.gamma[c] + h * 64 + g * 8);
      const float4* bt = reinterpret_cast<const float4*>(p.beta[c] + h * 64 + g * 8);
      const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1), b0 = __ldg(bt), b1 = __ldg(bt + 1);
      gg[0] = g0.x; gg[1] = g0.y; gg[2] = g0.z; gg[3] = g0.w;
      gg[4] = g1.x; gg[5] = g1.y; gg[6] = g1.z; gg[7] = g1.w;
      bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
      bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
    }
    const float mult = (c == 0) ? p.q_mult : 1.0f;
    const long long row_src = static_cast<long long>(idx) * 64 + g * 8;        // (c, h) inside the token block
    const long long row_dst = static_cast<long long>(h) * p.L * 64 + g * 8;    // head h of q/k
    const int j0 = 8 * (g & 1);
    const bool second = (g & 2) != 0;
    const int half = g < 4 ? 0 : 1;                 // 0: row rotation (dims 0-31), 1: column rotation
    for (int i0 = blockIdx.x; i0 < p.n_tok; i0 += TOKENS * gridDim.x) {
      PrologueToken w[TOKENS];
      uint4 raw[TOKENS];
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        const int ik = i0 + k * gridDim.x;
        w[k] = prologue_token(p, static_cast<uint32_t>(ik < p.n_tok ? ik : i0));
      }
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) raw[k] = *reinterpret_cast<const uint4*>(p.qkv + w[k].src + row_src);
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        if (i0 + k * static_cast<int>(gridDim.x) >= p.n_tok) continue;
        if (c == 2) {   // register-mode v gather: plain copy
          *reinterpret_cast<uint4*>(p.ws_v + w[k].dst_v + h * 64 + g * 8) = raw[k];
          continue;
        }
        float x[8];
        const uint32_t wd[4] = {raw[k].x, raw[k].y, raw[k].z, raw[k].w};
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
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = x[e] * rstd * gg[e] + bb[e];
        // 2D RoPE on patch tokens.  Lanes 0-3 hold dims 0-31 (row), 4-7 dims
        // 32-63 (col); lanes with bit 1 clear hold the first member j of a
        // pair (j, j+16), their partner is lane g^2.  The branch is uniform
        // over the 8-lane group, the shuffles run in every lane of the group.
        float partner[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) partner[e] = __shfl_xor_sync(gmask, x[e], 2);
        if (w[k].t >= p.n_special) {
          uint32_t pcol;
          const uint32_t prow = fast_divmod(static_cast<uint32_t>(w[k].t - p.n_special), p.div_gw, pcol);
          const int pos_idx = half == 0 ? static_cast<int>(prow) : p.grid_h + static_cast<int>(pcol);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float2 cs = rope_tab[pos_idx * 16 + j0 + e];
            x[e] = second ? (x[e] * cs.x + partner[e] * cs.y) : (x[e] * cs.x - partner[e] * cs.y);
          }
        }
        uint4 o;
        o.x = pack_bf16x2(x[0] * mult, x[1] * mult);
        o.y = pack_bf16x2(x[2] * mult, x[3] * mult);
        o.z = pack_bf16x2(x[4] * mult, x[5] * mult);
        o.w = pack_bf16x2(x[6] * mult, x[7] * mult);
        *reinterpret_cast<uint4*>(p.ws_qk[c] + w[k].dst_qk + row_dst) = o;
      }
    }
  }
}

}  // namespace vggt
