// Token LayerNorm of the transformer blocks around the attention core
// (VGGT-Omega Aggregator explainer, section 3: each frame and inter-frame
// block of a layer is a pre-norm transformer block; its norms work over the
// 1024 channels of a token): y = (x - mean) / sqrt(var + eps) * gamma + beta
// over the C values of a row, biased variance, fp32 arithmetic, bf16 in/out.
//
// HBM-bound (2 C bytes read + 2 C written per row).  One warp per row: lane l
// holds the 16-byte chunks l, l + 32, ... of the row (VPL of them, C = 256 VPL),
// so each load and store instruction of a warp covers 512 contiguous bytes;
// mean and variance (two passes over the registers) by butterfly shuffles.
// Warps stride over the rows; the grid is sized to the resident capacity.
#pragma once

#include <cstdint>

#include "common.cuh"

namespace vggt {

struct LayerNormParams {
  const uint16_t* x;     // [M][C] bf16
  uint16_t* y;           // [M][C] bf16 (may be x)
  const float* gamma;    // [C]
  const float* beta;     // [C]
  long long M;
  float eps;
  int* status;           // cleared by block 0 when zero_status (the first kernel of a block)
  int zero_status;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int VPL>
__global__ void __launch_bounds__(256) layernorm_rows_kernel(const LayerNormParams p) {
  constexpr int C = 256 * VPL;
  const int lane = threadIdx.x & 31;
  if (p.zero_status && blockIdx.x == 0 && threadIdx.x == 0) {
    p.status[0] = 0;
    p.status[1] = 0;
  }
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < p.M;
       r += warps) {
    const uint4* xr = reinterpret_cast<const uint4*>(p.x + r * C);
    float v[VPL][8];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const uint4 q = xr[lane + 32 * i];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[i][2 * k] = __uint_as_float(w[k] << 16);
        v[i][2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) s += v[i][e];
    const float mean = warp_sum(s) * (1.0f / C);
    float sq = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        v[i][e] -= mean;
        sq += v[i][e] * v[i][e];
      }
    const float rstd = rsqrtf(warp_sum(sq) * (1.0f / C) + p.eps);
    uint4* yr = reinterpret_cast<uint4*>(p.y + r * C);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int c0 = (lane + 32 * i) * 8;
      const float4 g0 = __ldg(reinterpret_cast<const float4*>(p.gamma + c0));
      const float4 g1 = __ldg(reinterpret_cast<const float4*>(p.gamma + c0 + 4));
      const float4 b0 = __ldg(reinterpret_cast<const float4*>(p.beta + c0));
      const float4 b1 = __ldg(reinterpret_cast<const float4*>(p.beta + c0 + 4));
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      float o[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = v[i][e] * rstd * g[e] + b[e];
      uint4 q;
      q.x = pack_bf16x2(o[0], o[1]);
      q.y = pack_bf16x2(o[2], o[3]);
      q.z = pack_bf16x2(o[4], o[5]);
      q.w = pack_bf16x2(o[6], o[7]);
      yr[lane + 32 * i] = q;
    }
  }
}

}  // namespace vggt
