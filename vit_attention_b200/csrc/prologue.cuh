// QK-LayerNorm + 2D RoPE prologue (VGGT-Omega Aggregator explainer,
// section 3: "use_qk_norm=True" and the 2D RoPE re-applied at every layer).
//
// Reads the q and k rows of the packed bf16 qkv[S][T][3][H][64], normalises
// each 64-dim head vector (biased variance, per-head affine), rotates patch
// tokens, multiplies q by softmax_scale*log2(e) (so the core works in base 2)
// and writes bf16 into the workspace in the attention core's layout
//   q, k : [H][B][L][64]   (frame: B = S, L = T; global: B = 1, L = S*T;
//                           register: B = 1, L = S*n_special), i.e. one
//                           [B*L][64] plane per head in the mode's token order
//   v    : [L][H][64]      (register mode only: the gathered special tokens)
//
// HBM-bound: 4 threads own one 128-byte head row.  Lane l of a row's group
// holds dims {b, .., b+7} and {b+16, .., b+23} with b = 32 (l / 2) + 8 (l % 2),
// so both members of every RoPE pair (j, j+16) of its half sit in the lane
// and the rotation needs no shuffle; the LayerNorm reductions are 2 shuffles
// inside the 4-lane group.  A block has one group per head row of a token
// (n_c*H groups, n_c*H*128 contiguous bytes of qkv), so a group keeps the same
// (tensor, head) for all the tokens it visits and holds that row's gamma/beta
// in registers; each lane keeps four tokens' loads in flight.  Token ->
// (problem, position, frame slot) divisions use a multiply-high by a
// precomputed reciprocal with one correction step.  The cos/sin table of
// every (row|col position, frequency) is built once per block in fp64 and
// kept in shared memory as fp32.
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

constexpr int PRO_MAX_THREADS = 256;   // 4 lanes per head row: 64 rows per block at most

struct PrologueParams {
  const uint16_t* qkv;
  const float* gamma[2];  // q, k
  const float* beta[2];
  uint16_t* ws_qk[2];     // q, k destinations
  uint16_t* ws_v;         // v copied token-major [L][H][64] when n_c == 3
  int k_token_major;      // k written token-major [L][H][64] (like v) instead of the head planes
  int* status;         // cleared by block 0 when zero_status (the first kernel of a call)
  int zero_status;
  long long qkv_elems;    // elements of qkv, of each q/k destination and of the v destination
  long long qk_elems, v_elems;   // (bounds of the debug build's checks)
  int n_tok;              // tokens in the mode's token list (< 2^31, checked on the host)
  int T, H, n_special, grid_h, grid_w;
  int mode;               // VGGT_ATTN_FRAME / GLOBAL / REGISTER
  int L;                  // tokens per problem in the workspace
  int n_c;                // 2 (q, k) or 3 (q, k and a copy of v: register mode, sharded global mode)
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
  w.dst_qk = (static_cast<long long>(b) * p.L + pos) * 64;
  w.dst_v = static_cast<long long>(pos) * p.H * 64;
  return w;
}

__global__ void __launch_bounds__(PRO_MAX_THREADS) qk_norm_rope_kernel(const PrologueParams p) {
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
  if (p.zero_status && blockIdx.x == 0 && threadIdx.x == 0) {
    p.status[0] = 0;
    p.status[1] = 0;
  }
  __syncthreads();

  const int l = threadIdx.x & 3;                    // lane inside the 4-lane row group
  // Shuffles involve only the 4 lanes of one row group: the groups of a warp
  // may take different paths (v rows, loop tail).
  const unsigned gmask = 0xFu << (threadIdx.x & 28);
  const int half = l >> 1;                          // 0: dims 0-31 rotate by row, 1: dims 32-63 by column
  const int base = 32 * half + 8 * (l & 1);         // first dim of the lane's first run of 8
  const int j0 = 8 * (l & 1);                       // RoPE frequency of the lane's first pair
  constexpr int TOKENS = 4;
  const int ch = p.n_c * p.H;
  const int groups = blockDim.x >> 2;
  for (int idx = threadIdx.x >> 2; idx < ch; idx += groups) {   // uniform over the 4-lane group
    const int c = idx / p.H, h = idx - c * p.H;
    float ga[8], gb[8], ba[8], bb[8];               // gamma/beta of the lane's two runs
    if (c < 2) {
      const float4* gm = reinterpret_cast<const float4*>(p.gamma[c] + h * 64 + base);
      const float4* bt = reinterpret_cast<const float4*>(p.beta[c] + h * 64 + base);
      const float4 g0 = __ldg(gm), g1 = __ldg(gm + 1), g2 = __ldg(gm + 4), g3 = __ldg(gm + 5);
      const float4 b0 = __ldg(bt), b1 = __ldg(bt + 1), b2 = __ldg(bt + 4), b3 = __ldg(bt + 5);
      ga[0] = g0.x; ga[1] = g0.y; ga[2] = g0.z; ga[3] = g0.w; ga[4] = g1.x; ga[5] = g1.y; ga[6] = g1.z; ga[7] = g1.w;
      gb[0] = g2.x; gb[1] = g2.y; gb[2] = g2.z; gb[3] = g2.w; gb[4] = g3.x; gb[5] = g3.y; gb[6] = g3.z; gb[7] = g3.w;
      ba[0] = b0.x; ba[1] = b0.y; ba[2] = b0.z; ba[3] = b0.w; ba[4] = b1.x; ba[5] = b1.y; ba[6] = b1.z; ba[7] = b1.w;
      bb[0] = b2.x; bb[1] = b2.y; bb[2] = b2.z; bb[3] = b2.w; bb[4] = b3.x; bb[5] = b3.y; bb[6] = b3.z; bb[7] = b3.w;
    }
    const float mult = (c == 0) ? p.q_mult : 1.0f;
    const long long row_src = static_cast<long long>(idx) * 64 + base;         // (c, h) inside the token block
    const long long row_dst = static_cast<long long>(h) * p.n_tok * 64 + base; // plane of head h
    for (int i0 = blockIdx.x; i0 < p.n_tok; i0 += TOKENS * gridDim.x) {
      PrologueToken w[TOKENS];
      uint4 ra[TOKENS], rb[TOKENS];
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        const int ik = i0 + k * gridDim.x;
        w[k] = prologue_token(p, static_cast<uint32_t>(ik < p.n_tok ? ik : i0));
      }
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        const uint16_t* src = p.qkv + w[k].src + row_src;
        if (VGGT_DBG_BOUNDS(w[k].src + row_src + 24 <= p.qkv_elems, p.status, 0x920u)) {
          ra[k] = *reinterpret_cast<const uint4*>(src);
          rb[k] = *reinterpret_cast<const uint4*>(src + 16);
        } else {
          ra[k] = rb[k] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int k = 0; k < TOKENS; ++k) {
        if (i0 + k * static_cast<int>(gridDim.x) >= p.n_tok) continue;
        if (c == 2) {   // register-mode v gather: plain copy
          uint16_t* dst = p.ws_v + w[k].dst_v + h * 64 + base;
          if (VGGT_DBG_BOUNDS(w[k].dst_v + h * 64 + base + 24 <= p.v_elems, p.status, 0x921u)) {
            *reinterpret_cast<uint4*>(dst) = ra[k];
            *reinterpret_cast<uint4*>(dst + 16) = rb[k];
          }
          continue;
        }
        float xa[8], xb[8];
        const uint32_t wa[4] = {ra[k].x, ra[k].y, ra[k].z, ra[k].w};
        const uint32_t wb[4] = {rb[k].x, rb[k].y, rb[k].z, rb[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          xa[2 * e] = __uint_as_float(wa[e] << 16);
          xa[2 * e + 1] = __uint_as_float(wa[e] & 0xFFFF0000u);
          xb[2 * e] = __uint_as_float(wb[e] << 16);
          xb[2 * e + 1] = __uint_as_float(wb[e] & 0xFFFF0000u);
        }
        // LayerNorm over the 64 values held by the 4-lane group (two passes).
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) sum += xa[e] + xb[e];
        sum += __shfl_xor_sync(gmask, sum, 1);
        sum += __shfl_xor_sync(gmask, sum, 2);
        const float mean = sum * (1.0f / 64.0f);
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          xa[e] -= mean;
          xb[e] -= mean;
          sq += xa[e] * xa[e] + xb[e] * xb[e];
        }
        sq += __shfl_xor_sync(gmask, sq, 1);
        sq += __shfl_xor_sync(gmask, sq, 2);
        const float rstd = rsqrtf(sq * (1.0f / 64.0f) + p.eps);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          xa[e] = xa[e] * rstd * ga[e] + ba[e];
          xb[e] = xb[e] * rstd * gb[e] + bb[e];
        }
        // 2D RoPE on patch tokens: pair (j, j+16) of the lane's half is
        // (xa[e], xb[e]) with j = j0 + e.
        if (w[k].t >= p.n_special) {
          uint32_t pcol;
          const uint32_t prow = fast_divmod(static_cast<uint32_t>(w[k].t - p.n_special), p.div_gw, pcol);
          const int pos_idx = half == 0 ? static_cast<int>(prow) : p.grid_h + static_cast<int>(pcol);
          const float4* cs4 = reinterpret_cast<const float4*>(rope_tab + pos_idx * 16 + j0);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float4 cs = cs4[e2];   // (cos, sin) of frequencies j0 + 2 e2 and j0 + 2 e2 + 1
            const float a0 = xa[2 * e2], b0 = xb[2 * e2], a1 = xa[2 * e2 + 1], b1 = xb[2 * e2 + 1];
            xa[2 * e2] = a0 * cs.x - b0 * cs.y;
            xb[2 * e2] = b0 * cs.x + a0 * cs.y;
            xa[2 * e2 + 1] = a1 * cs.z - b1 * cs.w;
            xb[2 * e2 + 1] = b1 * cs.z + a1 * cs.w;
          }
        }
        uint4 oa, ob;
        oa.x = pack_bf16x2(xa[0] * mult, xa[1] * mult);
        oa.y = pack_bf16x2(xa[2] * mult, xa[3] * mult);
        oa.z = pack_bf16x2(xa[4] * mult, xa[5] * mult);
        oa.w = pack_bf16x2(xa[6] * mult, xa[7] * mult);
        ob.x = pack_bf16x2(xb[0] * mult, xb[1] * mult);
        ob.y = pack_bf16x2(xb[2] * mult, xb[3] * mult);
        ob.z = pack_bf16x2(xb[4] * mult, xb[5] * mult);
        ob.w = pack_bf16x2(xb[6] * mult, xb[7] * mult);
        const long long dst_off = (c == 1 && p.k_token_major) ? w[k].dst_v + h * 64 + base : w[k].dst_qk + row_dst;
        uint16_t* dst = p.ws_qk[c] + dst_off;
        [[maybe_unused]] const long long dst_elems = (c == 1 && p.k_token_major) ? p.v_elems : p.qk_elems;
        if (VGGT_DBG_BOUNDS(dst_off + 24 <= dst_elems, p.status, 0x922u)) {
          *reinterpret_cast<uint4*>(dst) = oa;
          *reinterpret_cast<uint4*>(dst + 16) = ob;
        }
      }
    }
  }
}

}  // namespace vggt
