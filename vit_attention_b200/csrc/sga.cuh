// Subsampled global attention (AVGGT article, section B, point 2, "SGA"):
// keys/values are subsampled on the patch grid (one token per s_h x s_w
// window, every camera/register token kept), every query is kept, each token
// keeps its diagonal, and one mean key/value pair stands in for the discarded
// columns.  The QK-LayerNorm + RoPE prologue of global mode writes q and k of
// every token; these two kernels then gather the kept keys/values into dense
// arrays for the attention core and sum k and v over the discarded tokens
// (the core's epilogue adds the diagonal and the mean pair per row).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

struct SgaGeometry {
  int N, Nk, H, T, n_special, grid_w, s_h, s_w, nw, kept_per_frame;
  int grid_h;
};

// Flat token index (s*T + t) of the r-th kept key: frame r / kept_per_frame;
// inside it the n_special special tokens, then the kept patches row-major.
__device__ __forceinline__ int sga_kept_token(const SgaGeometry& g, int r) {
  const int s = r / g.kept_per_frame, u = r - s * g.kept_per_frame;
  int t = u;
  if (u >= g.n_special) {
    const int k = u - g.n_special;
    const int kr = k / g.nw, kc = k - kr * g.nw;
    t = g.n_special + kr * g.s_h * g.grid_w + kc * g.s_w;
  }
  return s * g.T + t;
}

__device__ __forceinline__ bool sga_is_kept(const SgaGeometry& g, int flat) {
  const int t = flat % g.T;
  if (t < g.n_special) return true;
  const int pp = t - g.n_special;
  const int prow = pp / g.grid_w, pcol = pp - prow * g.grid_w;
  return (prow % g.s_h == 0) && (pcol % g.s_w == 0);
}

// Kept keys (normalised k plane [H][N][64] -> [H][Nk][64]) and values
// (qkv [N][3][H][64] -> [Nk][H][64]); one block per kept token, 16 bytes per thread.
__global__ void __launch_bounds__(256) sga_gather_kernel(SgaGeometry g, const uint16_t* k_plane, const uint16_t* qkv,
                                                         uint16_t* ks_plane, uint16_t* vs) {
  for (int r = blockIdx.x; r < g.Nk; r += gridDim.x) {
    const int flat = sga_kept_token(g, r);
    for (int e = threadIdx.x; e < g.H * 8; e += blockDim.x) {
      const int h = e >> 3, c = e & 7;
      reinterpret_cast<uint4*>(ks_plane + (static_cast<size_t>(h) * g.Nk + r) * 64)[c] =
          reinterpret_cast<const uint4*>(k_plane + (static_cast<size_t>(h) * g.N + flat) * 64)[c];
      reinterpret_cast<uint4*>(vs + (static_cast<size_t>(r) * g.H + h) * 64)[c] =
          reinterpret_cast<const uint4*>(qkv + ((static_cast<size_t>(flat) * 3 + 2) * g.H + h) * 64)[c];
    }
  }
}

// sums[0][h][d] += k over the discarded tokens, sums[1][h][d] += v.  A block
// takes a contiguous range of tokens; thread e < 8H sums dims 8(e%8)..+7 of k
// of head e/8 (one 16-byte load per token: the head rows of a token are whole
// 128-byte lines), thread 8H + e the same dims of v; each thread adds its 8
// partial sums into `sums` once at the end.
__global__ void __launch_bounds__(256) sga_sum_kernel(SgaGeometry g, const uint16_t* k_plane, const uint16_t* qkv,
                                                      float* sums) {
  const int lanes = g.H * 8;                        // 16-byte chunks per token, for k and for v each
  const int per_block = (g.N + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * per_block;
  const int t1 = min(g.N, t0 + per_block);
  for (int e = threadIdx.x; e < 2 * lanes; e += blockDim.x) {
    const bool is_v = e >= lanes;
    const int c = is_v ? e - lanes : e;             // chunk: head c / 8, dims 8 (c % 8) ..
    const int h = c >> 3, d8 = c & 7;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int tok = t0; tok < t1; ++tok) {
      if (sga_is_kept(g, tok)) continue;            // the same for every thread of the block
      const uint4 w = is_v ? reinterpret_cast<const uint4*>(qkv + ((static_cast<size_t>(tok) * 3 + 2) * g.H + h) * 64)[d8]
                           : reinterpret_cast<const uint4*>(k_plane + (static_cast<size_t>(h) * g.N + tok) * 64)[d8];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc[2 * k] += __uint_as_float(ww[k] << 16);
        acc[2 * k + 1] += __uint_as_float(ww[k] & 0xFFFF0000u);
      }
    }
    float* dst = sums + (is_v ? g.H * 64 : 0) + h * 64 + d8 * 8;
#pragma unroll
    for (int k = 0; k < 8; ++k) atomicAdd(dst + k, acc[k]);
  }
}

// Descriptor attention (FlashVGGT article, abstract): descriptor r of a
// frame is one of its camera/register tokens, copied, or one s_h x s_w window
// of its patch grid (windows tile the grid from (0, 0), edge windows smaller)
// whose key is the mean of the window's normalised rotated keys and whose
// value is the mean of its values (fp32 sums, one bf16 rounding).  Keys go to
// [H][Nk][64], values to [Nk][H][64]; a block per descriptor, a thread per
// (head, pair of dims).
__global__ void __launch_bounds__(256) desc_pool_kernel(SgaGeometry g, const uint16_t* k_plane, const uint16_t* qkv,
                                                        uint16_t* ks_plane, uint16_t* vs) {
  for (int r = blockIdx.x; r < g.Nk; r += gridDim.x) {
    const int s = r / g.kept_per_frame, u = r - s * g.kept_per_frame;
    int r0 = 0, r1 = 1, c0 = 0, c1 = 1, t0 = u;     // special token: a 1 x 1 "window" at t0
    if (u >= g.n_special) {
      const int k = u - g.n_special;
      const int kr = k / g.nw, kc = k - kr * g.nw;
      r0 = kr * g.s_h;
      r1 = min(r0 + g.s_h, g.grid_h);
      c0 = kc * g.s_w;
      c1 = min(c0 + g.s_w, g.grid_w);
      t0 = g.n_special;
    }
    const float inv = 1.0f / static_cast<float>((r1 - r0) * (c1 - c0));
    for (int e = threadIdx.x; e < g.H * 32; e += blockDim.x) {
      const int h = e >> 5, d2 = e & 31;           // dims 2 d2, 2 d2 + 1 of head h
      float k0 = 0.f, k1 = 0.f, v0 = 0.f, v1 = 0.f;
      for (int rr = r0; rr < r1; ++rr)
        for (int cc = c0; cc < c1; ++cc) {
          const int tok = s * g.T + t0 + (u >= g.n_special ? rr * g.grid_w + cc : 0);
          const uint32_t kw = reinterpret_cast<const uint32_t*>(k_plane + (static_cast<size_t>(h) * g.N + tok) * 64)[d2];
          const uint32_t vw =
              reinterpret_cast<const uint32_t*>(qkv + ((static_cast<size_t>(tok) * 3 + 2) * g.H + h) * 64)[d2];
          k0 += __uint_as_float(kw << 16);
          k1 += __uint_as_float(kw & 0xFFFF0000u);
          v0 += __uint_as_float(vw << 16);
          v1 += __uint_as_float(vw & 0xFFFF0000u);
        }
      reinterpret_cast<uint32_t*>(ks_plane + (static_cast<size_t>(h) * g.Nk + r) * 64)[d2] = pack_bf16x2(k0 * inv, k1 * inv);
      reinterpret_cast<uint32_t*>(vs + (static_cast<size_t>(r) * g.H + h) * 64)[d2] = pack_bf16x2(v0 * inv, v1 * inv);
    }
  }
}

}  // namespace vggt
