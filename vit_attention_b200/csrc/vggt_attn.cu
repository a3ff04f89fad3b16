// Host side of libvggt_attn.so: argument validation, workspace layout, TMA
// tensor maps and the kernel launches behind the C ABI in vggt_attn.h.
//
// Sections, in order:
//   shape checks, workspace views, tensor maps, prologue / core launches
//   attention entry points (frame, global, register, prologue, core, status)
//   allocation-free entry point (static scratch)
//   projections: vggt_linear, vggt_attn_qkv_proj, vggt_attn_block
//   subsampled global attention (SGA) and descriptor attention
//   transformer blocks and the alternating layer schedule
//   camera-head trunk
//   query-sharded global attention (gathered form)
//   host-memory pipeline
//   query-sharded global attention (fused form: every rank's keys in place)
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attention_frame_persistent.cuh"
#include "attention_sm100.cuh"
#include "layernorm.cuh"
#include "linear_sm100.cuh"
#include "prologue.cuh"
#include "sga.cuh"
#include "vggt_attn.h"

namespace {

using vggt::kStatusBytes;

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait; no wait in a healthy run is near it
constexpr int kMaxRopePositions = 3000;                           // grid_h + grid_w (cos/sin table in shared memory)

struct ModeGeometry {
  long long B;      // independent problems
  long long L;      // tokens per problem
  long long n_tok;  // tokens the prologue handles
  int n_c;          // head rows per token the prologue handles (q, k[, v])
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool valid_mode(int mode) { return mode == VGGT_ATTN_FRAME || mode == VGGT_ATTN_GLOBAL || mode == VGGT_ATTN_REGISTER; }

int check_shape(const vggt_attn_shape* s, int mode) {
  if (!s || !valid_mode(mode)) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(s->ln_eps) || !std::isfinite(s->rope_base) || !std::isfinite(s->softmax_scale))
    return VGGT_ATTN_ERR_INVALID_ARG;
  if (!(s->ln_eps > 0.f) || !(s->rope_base > 0.f)) return VGGT_ATTN_ERR_INVALID_ARG;
  if (s->head_dim != 64) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (s->S < 1 || s->T < 1 || s->H < 1 || s->n_special < 0 || s->n_special > s->T || s->grid_h < 0 ||
      s->grid_w < 0)
    return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<long long>(s->n_special) + static_cast<long long>(s->grid_h) * s->grid_w != s->T)
    return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (s->T > s->n_special && s->grid_w < 1) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (s->grid_h + static_cast<long long>(s->grid_w) > kMaxRopePositions) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (mode == VGGT_ATTN_REGISTER && s->n_special < 1) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (s->H > 65535) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;  // grid.y
  const long long n = static_cast<long long>(s->S) * s->T;
  if (n > (1LL << 31) - 1 - 256) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;  // int token indices in the core
  if (n * 3 * s->H > (1LL << 31) - 1) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;  // int row indices in the prologue
  if (mode == VGGT_ATTN_FRAME &&
      (static_cast<long long>(s->T) + 127) / 128 * s->H * s->S > INT32_MAX)   // int unit indices of the frame core
    return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  return VGGT_ATTN_OK;
}

ModeGeometry geometry(const vggt_attn_shape* s, int mode) {
  ModeGeometry g;
  const long long n = static_cast<long long>(s->S) * s->T;
  switch (mode) {
    case VGGT_ATTN_FRAME: g = {s->S, s->T, n, 2}; break;
    case VGGT_ATTN_GLOBAL: g = {1, n, n, 2}; break;
    default: g = {1, static_cast<long long>(s->S) * s->n_special, static_cast<long long>(s->S) * s->n_special, 3};
  }
  return g;
}

struct WorkspaceView {
  int* status;
  uint16_t* q;
  uint16_t* k;
  uint16_t* v;  // register mode only
  size_t bytes;
};

WorkspaceView workspace_view(const vggt_attn_shape* s, int mode, void* ws) {
  const ModeGeometry g = geometry(s, mode);
  const size_t qk_bytes = align256(static_cast<size_t>(g.B * g.L) * s->H * 64 * 2);
  WorkspaceView w;
  uint8_t* base = static_cast<uint8_t*>(ws);
  w.status = reinterpret_cast<int*>(base);
  w.q = reinterpret_cast<uint16_t*>(base + kStatusBytes);
  w.k = reinterpret_cast<uint16_t*>(base + kStatusBytes + qk_bytes);
  size_t total = kStatusBytes + 2 * qk_bytes;
  w.v = nullptr;
  if (mode == VGGT_ATTN_REGISTER) {
    w.v = reinterpret_cast<uint16_t*>(base + total);
    total += align256(static_cast<size_t>(g.L) * s->H * 64 * 2);
  }
  w.bytes = total;
  return w;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_device() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  if (major != 10 || minor != 0) return VGGT_ATTN_ERR_UNSUPPORTED_DEVICE;
  return VGGT_ATTN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor map, 128-byte swizzle, box inner dim 64 (= 128 B), zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides_bytes,
              const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides_bytes, box,
            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// clear_status: the prologue is the call's first kernel (the attention entry
// points); inside a block an earlier kernel has cleared the status word and
// may already have recorded an error in it.  shard_k / shard_v (global mode,
// one rank's frames): k and a copy of v go token-major ([L][H][64]) to these
// buffers, the ones all ranks gather, instead of k to the workspace plane.
int launch_prologue(int mode, const vggt_attn_shape* s, const void* qkv, const float* gq, const float* bq,
                    const float* gk, const float* bk, const WorkspaceView& w, cudaStream_t stream,
                    bool clear_status = true, uint16_t* shard_k = nullptr, uint16_t* shard_v = nullptr) {
  const ModeGeometry g = geometry(s, mode);
  vggt::PrologueParams p;
  p.qkv = static_cast<const uint16_t*>(qkv);
  p.gamma[0] = gq;
  p.gamma[1] = gk;
  p.beta[0] = bq;
  p.beta[1] = bk;
  p.ws_qk[0] = w.q;
  p.ws_qk[1] = w.k;
  p.ws_v = w.v;
  p.k_token_major = 0;
  p.n_c = g.n_c;
  if (shard_k) {
    p.ws_qk[1] = shard_k;
    p.ws_v = shard_v;
    p.k_token_major = 1;
    p.n_c = 3;
  }
  p.status = w.status;
  p.zero_status = clear_status ? 1 : 0;
  p.qkv_elems = static_cast<long long>(s->S) * s->T * 3 * s->H * 64;
  p.qk_elems = g.B * g.L * s->H * 64;
  p.v_elems = g.L * s->H * 64;
  p.n_tok = static_cast<int>(g.n_tok);
  p.T = s->T;
  p.H = s->H;
  p.n_special = s->n_special;
  p.grid_h = s->grid_h;
  p.grid_w = s->grid_w;
  p.mode = mode;
  p.L = static_cast<int>(g.L);
  p.div_nspec = vggt::make_fastdiv(static_cast<uint32_t>(s->n_special));
  p.div_L = vggt::make_fastdiv(static_cast<uint32_t>(g.L));
  p.div_T = vggt::make_fastdiv(static_cast<uint32_t>(s->T));
  p.div_gw = vggt::make_fastdiv(static_cast<uint32_t>(s->grid_w > 0 ? s->grid_w : 1));
  p.eps = s->ln_eps;
  const double scale = s->softmax_scale > 0.f ? static_cast<double>(s->softmax_scale) : 1.0 / std::sqrt(64.0);
  p.q_mult = static_cast<float>(scale * 1.4426950408889634);  // log2(e)
  p.rope_base = s->rope_base;

  // One 4-lane group per head row of a token (a group loops over rows when a
  // token has more than 64); as many blocks as fit on the device at once,
  // each striding over the tokens four at a time.
  const int ch = p.n_c * s->H;
  const int threads = ch <= 64 ? 4 * ch : 256;
  const size_t smem = static_cast<size_t>(s->grid_h + s->grid_w) * 16 * sizeof(float2);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(vggt::qk_norm_rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, vggt::qk_norm_rope_kernel, threads, smem) !=
          cudaSuccess || per_sm < 1)
    return VGGT_ATTN_ERR_CUDA;
  long long blocks = static_cast<long long>(sms) * per_sm;
  if (blocks > g.n_tok) blocks = g.n_tok;
  if (blocks < 1) blocks = 1;
  vggt::qk_norm_rope_kernel<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

template <class C>
int launch_core_cfg(const ModeGeometry& g, int H, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const vggt::CoreParams& p, cudaStream_t stream) {
  if (cudaFuncSetAttribute(vggt::attn_core_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC) !=
      cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  // The kernel re-splits its registers between warpgroups (setmaxnreg); that
  // split assumes the compiled per-thread count.  A build with fewer registers
  // at launch would make the softmax warps wait forever for registers, so
  // refuse to launch it.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, vggt::attn_core_kernel<C>) != cudaSuccess || fa.numRegs < C::REGS_AT_LAUNCH)
    return VGGT_ATTN_ERR_CUDA;
  constexpr int rows_per_cta = vggt::core::BM * C::NQ;
  const long long n_q = (g.L + rows_per_cta - 1) / rows_per_cta;
  const dim3 grid(static_cast<unsigned>(n_q), static_cast<unsigned>(H), static_cast<unsigned>(g.B));
  vggt::attn_core_kernel<C><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

// Frame mode: persistent CTAs, two per SM, each walking the (tile, head,
// frame) units with a stride of the grid size.
int launch_frame_persistent(const ModeGeometry& g, int H, const CUtensorMap& mq, const CUtensorMap& mk,
                            const CUtensorMap& mv, const vggt::CoreParams& p, cudaStream_t stream) {
  // output tile map: out[S][T][H][64] as (dim, head, token, frame), one 128-token box per store
  CUtensorMap mo;
  {
    const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(g.L),
                                static_cast<cuuint64_t>(g.B)};
    const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(H) * 128 * g.L};
    const cuuint32_t box[4] = {64, 1, vggt::core::BM, 1};
    if (!make_map(&mo, p.out, 4, dims, strides, box)) return VGGT_ATTN_ERR_CUDA;
  }
  if (cudaFuncSetAttribute(vggt::attn_frame_persistent_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           vggt::fp::SMEM_ALLOC) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  cudaFuncAttributes fa;   // the register split assumes the compiled count (see launch_core_cfg)
  if (cudaFuncGetAttributes(&fa, vggt::attn_frame_persistent_kernel) != cudaSuccess ||
      fa.numRegs < vggt::fp::REGS_AT_LAUNCH)
    return VGGT_ATTN_ERR_CUDA;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  vggt::FrameUnits fu;
  fu.n_qt = static_cast<int>((g.L + vggt::core::BM - 1) / vggt::core::BM);
  const long long n_units = static_cast<long long>(fu.n_qt) * H * g.B;   // < 2^31: checked with the shape
  fu.n_units = static_cast<int>(n_units);
  long long grid = static_cast<long long>(sms) * vggt::fp::CTAS_PER_SM;
  if (grid > n_units) grid = n_units;
  vggt::attn_frame_persistent_kernel<<<static_cast<unsigned>(grid), vggt::fp::THREADS, vggt::fp::SMEM_ALLOC,
                                       stream>>>(mq, mk, mv, mo, p, fu);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

int launch_core(int mode, const vggt_attn_shape* s, const void* qkv, void* out, const WorkspaceView& w,
                cudaStream_t stream) {
  const ModeGeometry g = geometry(s, mode);
  CUtensorMap mq, mk, mv;
  // keys per step: 80 in the frame kernel, 64 in the others
  const cuuint32_t kv_rows = mode == VGGT_ATTN_FRAME ? vggt::fp::BN : vggt::core::BN;
  {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(g.L), static_cast<cuuint64_t>(g.B * s->H)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(g.L) * 128};
    const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};   // one query tile
    const cuuint32_t box_k[3] = {64, kv_rows, 1};          // one key tile
    if (!make_map(&mq, w.q, 3, dims, strides, box_q) || !make_map(&mk, w.k, 3, dims, strides, box_k))
      return VGGT_ATTN_ERR_CUDA;
  }
  {
    const cuuint32_t box[4] = {64, 1, kv_rows, 1};         // one value tile
    if (mode == VGGT_ATTN_REGISTER) {  // gathered v: [L][H][64]
      const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(s->H), static_cast<cuuint64_t>(g.L), 1};
      const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(s->H) * 128,
                                     static_cast<cuuint64_t>(g.L) * s->H * 128};
      if (!make_map(&mv, w.v, 4, dims, strides, box)) return VGGT_ATTN_ERR_CUDA;
    } else {  // v straight from qkv[S][T][3][H][64]: (dim, head, token, problem)
      const cuuint64_t tok = static_cast<cuuint64_t>(3) * s->H * 128;
      const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(s->H), static_cast<cuuint64_t>(g.L),
                                  static_cast<cuuint64_t>(g.B)};
      const cuuint64_t strides[3] = {128, tok, tok * static_cast<cuuint64_t>(g.L)};
      const uint8_t* vbase = static_cast<const uint8_t*>(qkv) + static_cast<size_t>(2) * s->H * 128;
      if (!make_map(&mv, vbase, 4, dims, strides, box)) return VGGT_ATTN_ERR_CUDA;
    }
  }
  vggt::CoreParams p{};
  p.L = static_cast<int>(g.L);
  p.Lk = static_cast<int>(g.L);
  p.H = s->H;
  p.B = static_cast<int>(g.B);
  p.out_T = s->T;
  p.out_group = mode == VGGT_ATTN_REGISTER ? s->n_special : static_cast<int>(g.L);
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = static_cast<long long>(s->S) * s->T * s->H * 64;
  p.status = w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  // Frame mode: one query tile per CTA, two CTAs per SM; global and register
  // mode: two query tiles per CTA sharing every K/V tile.
  if (mode == VGGT_ATTN_FRAME) return launch_frame_persistent(g, s->H, mq, mk, mv, p, stream);
  return launch_core_cfg<vggt::CoreCfg<2>>(g, s->H, mq, mk, mv, p, stream);
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int check_common(int mode, const vggt_attn_shape* s, const void* qkv, void* ws, size_t ws_bytes) {
  int rc = check_shape(s, mode);
  if (rc) return rc;
  if (!qkv || !ws) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(ws, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  if (ws_bytes < vggt_attn_workspace_size(s, mode)) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  return VGGT_ATTN_OK;
}

int check_prologue_args(int mode, const vggt_attn_shape* s, const void* qkv, const float* gq, const float* bq,
                        const float* gk, const float* bk, void* ws, size_t ws_bytes) {
  int rc = check_common(mode, s, qkv, ws, ws_bytes);
  if (rc) return rc;
  if (!gq || !bq || !gk || !bk) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(gq, 16) || !aligned(bq, 16) || !aligned(gk, 16) || !aligned(bk, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  const size_t qkv_bytes = static_cast<size_t>(s->S) * s->T * 3 * s->H * 64 * 2;
  if (overlaps(ws, ws_bytes, qkv, qkv_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

int check_core_args(int mode, const vggt_attn_shape* s, const void* qkv, void* out, void* ws, size_t ws_bytes) {
  int rc = check_common(mode, s, qkv, ws, ws_bytes);
  if (rc) return rc;
  if (!out) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  const size_t qkv_bytes = static_cast<size_t>(s->S) * s->T * 3 * s->H * 64 * 2;
  const size_t out_bytes = static_cast<size_t>(s->S) * s->T * s->H * 64 * 2;
  if (overlaps(out, out_bytes, qkv, qkv_bytes) || overlaps(out, out_bytes, ws, ws_bytes))
    return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

int run_mode(int mode, const vggt_attn_shape* s, const void* qkv, const float* gq, const float* bq, const float* gk,
             const float* bk, void* out, void* ws, size_t ws_bytes, void* stream) {
  int rc = check_prologue_args(mode, s, qkv, gq, bq, gk, bk, ws, ws_bytes);
  if (rc) return rc;
  rc = check_core_args(mode, s, qkv, out, ws, ws_bytes);
  if (rc) return rc;
  if ((rc = check_device())) return rc;
  const WorkspaceView w = workspace_view(s, mode, ws);
  rc = launch_prologue(mode, s, qkv, gq, bq, gk, bk, w, static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  return launch_core(mode, s, qkv, out, w, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

size_t vggt_attn_workspace_size(const vggt_attn_shape* shape, int mode) {
  if (check_shape(shape, mode) != VGGT_ATTN_OK) return 0;
  return workspace_view(shape, mode, nullptr).bytes;
}

int vggt_attn_frame(const vggt_attn_shape* shape, const void* qkv, const float* q_gamma, const float* q_beta,
                    const float* k_gamma, const float* k_beta, void* out, void* workspace, size_t workspace_bytes,
                    void* cuda_stream) {
  return run_mode(VGGT_ATTN_FRAME, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes,
                  cuda_stream);
}

int vggt_attn_global(const vggt_attn_shape* shape, const void* qkv, const float* q_gamma, const float* q_beta,
                     const float* k_gamma, const float* k_beta, void* out, void* workspace, size_t workspace_bytes,
                     void* cuda_stream) {
  return run_mode(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes,
                  cuda_stream);
}

int vggt_attn_register(const vggt_attn_shape* shape, const void* qkv, const float* q_gamma, const float* q_beta,
                       const float* k_gamma, const float* k_beta, void* out, void* workspace, size_t workspace_bytes,
                       void* cuda_stream) {
  return run_mode(VGGT_ATTN_REGISTER, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace,
                  workspace_bytes, cuda_stream);
}

int vggt_attn_prologue(int mode, const vggt_attn_shape* shape, const void* qkv, const float* q_gamma,
                       const float* q_beta, const float* k_gamma, const float* k_beta, void* workspace,
                       size_t workspace_bytes, void* cuda_stream) {
  int rc = check_prologue_args(mode, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace, workspace_bytes);
  if (rc) return rc;
  if ((rc = check_device())) return rc;
  return launch_prologue(mode, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace_view(shape, mode, workspace),
                         static_cast<cudaStream_t>(cuda_stream));
}

int vggt_attn_core(int mode, const vggt_attn_shape* shape, const void* qkv, void* out, void* workspace,
                   size_t workspace_bytes, void* cuda_stream) {
  int rc = check_core_args(mode, shape, qkv, out, workspace, workspace_bytes);
  if (rc) return rc;
  if ((rc = check_device())) return rc;
  return launch_core(mode, shape, qkv, out, workspace_view(shape, mode, workspace),
                     static_cast<cudaStream_t>(cuda_stream));
}

int vggt_attn_read_status(void* workspace, void* cuda_stream, int* status) {
  if (!workspace || !status) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  vggt::StatusBlock host{0, 0};
  if (cudaMemcpyAsync(&host, workspace, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(host), st) != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  *status = host.code;
  return VGGT_ATTN_OK;
}

int vggt_attn_selftest_timeout(void* workspace, unsigned timeout_us, void* cuda_stream) {
  if (!workspace) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  if (timeout_us < 1 || timeout_us > 1000000) return VGGT_ATTN_ERR_INVALID_ARG;
  int rc = check_device();
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(vggt::StatusBlock), st) != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  vggt::selftest_timeout_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace), 1000ull * timeout_us);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

const char* vggt_attn_error_string(int code) {
  switch (code) {
    case VGGT_ATTN_OK: return "ok";
    case VGGT_ATTN_ERR_INVALID_ARG: return "invalid argument (null pointer, bad mode, overlapping buffers or bad scalar)";
    case VGGT_ATTN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape (head_dim must be 64, T == n_special + grid_h*grid_w, sizes in range)";
    case VGGT_ATTN_ERR_MISALIGNED: return "misaligned pointer (qkv/out/gamma/beta need 16 bytes, workspace 256 bytes)";
    case VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than vggt_attn_workspace_size()";
    case VGGT_ATTN_ERR_CUDA: return "CUDA runtime, driver or launch error";
    case VGGT_ATTN_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
    case VGGT_ATTN_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
    case VGGT_ATTN_ERR_SCRATCH_TOO_SMALL: return "problem needs more workspace than the fixed 64 MiB scratch of vggt_attn_noalloc";
    case VGGT_ATTN_ERR_BOUNDS: return "a device-side bounds check of the debug build failed (the access was skipped)";
    default: return "unknown error code";
  }
}

int vggt_attn_abi_version(void) { return VGGT_ATTN_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point.  For callers that cannot allocate device
// memory (plug-in interfaces that pass only inputs and outputs, code that must
// not call cudaMalloc/cudaFree, fixed device-memory budgets): the workspace is
// this file-scope array, which every GPU that loads the library holds until
// the process exits.  In host code `noalloc_scratch` names a host-side stand-in,
// not the device memory, so its device address is looked up with
// cudaGetSymbolAddress (with the device current) and only that address is
// passed to the kernels.
namespace {

static __device__ __align__(256) unsigned char noalloc_scratch[VGGT_ATTN_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex noalloc_mutex;
// Per device: the address and the CUDA context it belongs to.  A device reset
// (cudaDeviceReset) destroys the primary context and with it the module that
// holds the array; the next runtime call creates a new context with a new id,
// so the address is looked up again instead of reusing a dangling one.
struct NoallocSlot {
  unsigned long long ctx_id;
  void* ptr;
};
NoallocSlot noalloc_slot[kMaxDevices] = {};

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static PfnCtxGetCurrent get_current = nullptr;
  static PfnCtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PfnCtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PfnCtxGetId>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device, looked up the
// first time a context of that device calls (set-up), with that device current.
int noalloc_scratch_address(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VGGT_ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(noalloc_mutex);
  NoallocSlot& slot = noalloc_slot[dev];
  const unsigned long long ctx = current_context_id();   // 0 before the runtime has made a context current
  if (!slot.ptr || ctx == 0 || slot.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || p == nullptr) return VGGT_ATTN_ERR_CUDA;
    slot.ptr = p;
    slot.ctx_id = current_context_id();                   // the context the lookup ran in
  }
  *ptr = slot.ptr;
  return VGGT_ATTN_OK;
}

}  // namespace

extern "C" int vggt_attn_noalloc(int mode, const vggt_attn_shape* shape, const void* qkv, const float* q_gamma,
                                 const float* q_beta, const float* k_gamma, const float* k_beta, void* out,
                                 void* cuda_stream) {
  int rc = check_shape(shape, mode);
  if (rc) return rc;
  if (vggt_attn_workspace_size(shape, mode) > VGGT_ATTN_NOALLOC_SCRATCH_BYTES) return VGGT_ATTN_ERR_SCRATCH_TOO_SMALL;
  if ((rc = check_device())) return rc;
  void* scratch = nullptr;
  if ((rc = noalloc_scratch_address(&scratch))) return rc;
  return run_mode(mode, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, scratch, VGGT_ATTN_NOALLOC_SCRATCH_BYTES,
                  cuda_stream);
}


// ---------------------------------------------------------------------------
// Projections either side of the attention core: Y = X W^T + b, and the QKV
// projection with the QK LayerNorm + RoPE in its epilogue.
namespace {

bool make_rows_map(CUtensorMap* map, const void* base, long long inner, long long rows, cuuint32_t box_rows) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), 1};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner) * 2, static_cast<cuuint64_t>(inner) * 2 * rows};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(vggt::lin::BK), box_rows, 1};
  return make_map(map, base, 3, dims, strides, box);
}

int check_linear_dims(long long M, long long N, long long K) {
  if (M < 1 || N < vggt::lin::BN || K < vggt::lin::BK) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (N % vggt::lin::BN || K % vggt::lin::BK) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (M > (1LL << 30) || N > 65536 || K > 65536) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  return VGGT_ATTN_OK;
}

// Output maps: o0 = y [M][N] (plain) or the v slot of qkv [M][3][H][64]
// (qkv epilogue, as (64, H, 3, M)); o1, o2 = the q and k planes [H][M][64] (qkv epilogue).
template <int EPI>
int launch_linear_epi(const vggt::LinearParams& p, const CUtensorMap& mx, const CUtensorMap& mw, const CUtensorMap& o0,
                      const CUtensorMap& o1, const CUtensorMap& o2, int smem, unsigned grid, cudaStream_t stream) {
  static_assert(vggt::linear_smem_bytes(0, 0, vggt::lin::EPI_GELU) <= 227 * 1024, "two staging buffers fit");
  if (cudaFuncSetAttribute(vggt::linear_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  vggt::linear_kernel<EPI><<<grid, vggt::lin::threads_for(EPI), smem, stream>>>(mx, mw, o0, o1, o2, p);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

int launch_linear(vggt::LinearParams p, const void* x, const void* w, const CUtensorMap& o0, const CUtensorMap& o1,
                  const CUtensorMap& o2, int grid_h, int grid_w, cudaStream_t stream, int epi = vggt::lin::EPI_STD) {
  CUtensorMap mx, mw;
  if (!make_rows_map(&mx, x, p.K, p.M, vggt::lin::BM) || !make_rows_map(&mw, w, p.K, p.N, vggt::lin::BN))
    return VGGT_ATTN_ERR_CUDA;
  const int smem = vggt::linear_smem_bytes(grid_h, grid_w, epi);
  if (smem > 227 * 1024) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return VGGT_ATTN_ERR_CUDA;
  const long long tiles = ((p.M + vggt::lin::BM - 1) / vggt::lin::BM) * static_cast<long long>(p.N / vggt::lin::BN);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);   // persistent: one CTA per SM
  p.timeout_ns = kDefaultTimeoutNs;
  switch (epi) {
    case vggt::lin::EPI_GELU: return launch_linear_epi<vggt::lin::EPI_GELU>(p, mx, mw, o0, o1, o2, smem, grid, stream);
    case vggt::lin::EPI_RESID: return launch_linear_epi<vggt::lin::EPI_RESID>(p, mx, mw, o0, o1, o2, smem, grid, stream);
    case vggt::lin::EPI_QKV: return launch_linear_epi<vggt::lin::EPI_QKV>(p, mx, mw, o0, o1, o2, smem, grid, stream);
    default: return launch_linear_epi<vggt::lin::EPI_STD>(p, mx, mw, o0, o1, o2, smem, grid, stream);
  }
}

int check_qkv_proj_args(int mode, const vggt_attn_shape* s, const void* x, const void* w, const float* b,
                        const float* gq, const float* bq, const float* gk, const float* bk, void* qkv, void* ws,
                        size_t ws_bytes) {
  if (mode != VGGT_ATTN_FRAME && mode != VGGT_ATTN_GLOBAL) return VGGT_ATTN_ERR_INVALID_ARG;
  int rc = check_common(mode, s, qkv, ws, ws_bytes);
  if (rc) return rc;
  if (!x || !w || !gq || !bq || !gk || !bk) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w, 16) || (b && !aligned(b, 16)) || !aligned(gq, 16) || !aligned(bq, 16) ||
      !aligned(gk, 16) || !aligned(bk, 16))
    return VGGT_ATTN_ERR_MISALIGNED;
  const long long C = static_cast<long long>(s->H) * 64;
  if ((rc = check_linear_dims(static_cast<long long>(s->S) * s->T, 3 * C, C))) return rc;
  const size_t qkv_bytes = static_cast<size_t>(s->S) * s->T * 3 * C * 2;
  const size_t x_bytes = static_cast<size_t>(s->S) * s->T * C * 2;
  if (overlaps(qkv, qkv_bytes, x, x_bytes) || overlaps(ws, ws_bytes, x, x_bytes) ||
      overlaps(qkv, qkv_bytes, w, static_cast<size_t>(3 * C * C * 2)))
    return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

int launch_qkv_proj(int mode, const vggt_attn_shape* s, const void* x, const void* w, const float* b,
                    const float* gq, const float* bq, const float* gk, const float* bk, void* qkv,
                    const WorkspaceView& wv, cudaStream_t stream, bool zero_status = true) {
  const ModeGeometry g = geometry(s, mode);
  vggt::LinearParams p{};
  p.M = s->S * s->T;
  p.N = 3 * s->H * 64;
  p.K = s->H * 64;
  p.bias = b;
  p.status = wv.status;
  p.zero_status = zero_status ? 1 : 0;
  p.gamma[0] = gq;
  p.gamma[1] = gk;
  p.beta[0] = bq;
  p.beta[1] = bk;
  p.H = s->H;
  p.T = s->T;
  p.n_special = s->n_special;
  p.grid_h = s->grid_h;
  p.grid_w = s->grid_w > 0 ? s->grid_w : 1;
  p.eps = s->ln_eps;
  const double scale = s->softmax_scale > 0.f ? static_cast<double>(s->softmax_scale) : 1.0 / std::sqrt(64.0);
  p.q_mult = static_cast<float>(scale * 1.4426950408889634);  // log2(e)
  p.rope_base = s->rope_base;
  CUtensorMap mv, mq, mk;
  const long long M = p.M, H = s->H;
  {
    const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), 3, static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(3 * H) * 128};
    const cuuint32_t box[4] = {64, 1, 1, vggt::lin::BM};
    if (!make_map(&mv, qkv, 4, dims, strides, box)) return VGGT_ATTN_ERR_CUDA;
  }
  {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(H)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(M) * 128};
    const cuuint32_t box[3] = {64, vggt::lin::BM, 1};
    if (!make_map(&mq, wv.q, 3, dims, strides, box) || !make_map(&mk, wv.k, 3, dims, strides, box))
      return VGGT_ATTN_ERR_CUDA;
  }
  (void)g;
  return launch_linear(p, x, w, mv, mq, mk, s->grid_h, s->grid_w, stream, vggt::lin::EPI_QKV);
}

// The QKV projection of an attention block with the QK-LayerNorm + RoPE:
// the GEMM with the normalising epilogue (q and k straight into the
// workspace planes, v into its slot of qkv; measured 4-8 % faster than the
// plain GEMM followed by the prologue pass, which it replaces) when its
// cos/sin table fits in shared memory beside the GEMM's buffers, else the
// GEMM followed by the prologue.  zero_status: this is the call's first
// kernel.
int launch_block_qkv(int mode, const vggt_attn_shape* s, const void* x, const void* w, const float* b,
                     const float* gq, const float* bq, const float* gk, const float* bk, void* qkv,
                     const WorkspaceView& wv, cudaStream_t stream, bool zero_status);

}  // namespace

extern "C" int vggt_linear(int M, int N, int K, const void* x, const void* w, const float* bias, void* y,
                           void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_linear_dims(M, N, K);
  if (rc) return rc;
  if (!x || !w || !y || !workspace) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16) || (bias && !aligned(bias, 16)) ||
      !aligned(workspace, 256))
    return VGGT_ATTN_ERR_MISALIGNED;
  if (workspace_bytes < vggt::kStatusBytes) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  const size_t y_bytes = static_cast<size_t>(M) * N * 2;
  if (overlaps(y, y_bytes, x, static_cast<size_t>(M) * K * 2) || overlaps(y, y_bytes, w, static_cast<size_t>(N) * K * 2) ||
      overlaps(y, y_bytes, workspace, vggt::kStatusBytes))
    return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  vggt::LinearParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.bias = bias;
  p.status = static_cast<int*>(workspace);
  p.grid_h = 0;
  p.grid_w = 1;
  CUtensorMap my;
  if (!make_rows_map(&my, y, N, M, vggt::lin::BM)) return VGGT_ATTN_ERR_CUDA;
  return launch_linear(p, x, w, my, my, my, 0, 0, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" int vggt_attn_qkv_proj(int mode, const vggt_attn_shape* shape, const void* x, const void* w_qkv,
                                  const float* b_qkv, const float* q_gamma, const float* q_beta, const float* k_gamma,
                                  const float* k_beta, void* qkv, void* workspace, size_t workspace_bytes,
                                  void* cuda_stream) {
  int rc = check_qkv_proj_args(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, qkv, workspace,
                               workspace_bytes);
  if (rc) return rc;
  if ((rc = check_device())) return rc;
  return launch_qkv_proj(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, qkv,
                         workspace_view(shape, mode, workspace), static_cast<cudaStream_t>(cuda_stream));
}

namespace {

// Rows of the special tokens of every frame: compact row r <-> token row
// (r / n_special) * T + r % n_special.  to_compact: token rows -> compact rows.
__global__ void __launch_bounds__(128) special_rows_kernel(const uint4* src, uint4* dst, int n_rows, int row_vec,
                                                           int n_special, int T, int to_compact) {
  for (int r = blockIdx.x; r < n_rows; r += gridDim.x) {
    const long long tok = static_cast<long long>(r / n_special) * T + r % n_special;
    const long long from = to_compact ? tok : r, to = to_compact ? r : tok;
    for (int e = threadIdx.x; e < row_vec; e += blockDim.x)
      dst[to * row_vec + e] = src[from * row_vec + e];
  }
}

int launch_special_rows(const void* src, void* dst, int n_rows, long long row_bytes, int n_special, int T,
                        bool to_compact, cudaStream_t st) {
  const int grid = n_rows < 4096 ? n_rows : 4096;
  special_rows_kernel<<<grid, 128, 0, st>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n_rows,
                                            static_cast<int>(row_bytes / 16), n_special, T, to_compact ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

// y = epi(x w^T + b) into y [M][N]; EPI_RESID reads resid [M][N] and ls [N].
int launch_linear_plain(const void* x, const void* w, const float* b, void* y, long long M, long long N, long long K,
                        int* status, cudaStream_t st, bool zero_status = false, int epi = vggt::lin::EPI_STD,
                        const void* resid = nullptr, const float* ls = nullptr) {
  vggt::LinearParams p{};
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.bias = b;
  p.status = status;
  p.zero_status = zero_status ? 1 : 0;
  p.grid_w = 1;
  p.resid = static_cast<const uint16_t*>(resid);
  p.ls = ls;
  CUtensorMap my;
  if (!make_rows_map(&my, y, N, M, vggt::lin::BM)) return VGGT_ATTN_ERR_CUDA;
  return launch_linear(p, x, w, my, my, my, 0, 0, st, epi);
}

int launch_block_qkv(int mode, const vggt_attn_shape* s, const void* x, const void* w, const float* b,
                     const float* gq, const float* bq, const float* gk, const float* bk, void* qkv,
                     const WorkspaceView& wv, cudaStream_t stream, bool zero_status) {
  if (vggt::linear_smem_bytes(s->grid_h, s->grid_w, vggt::lin::EPI_QKV) <= 227 * 1024)
    return launch_qkv_proj(mode, s, x, w, b, gq, bq, gk, bk, qkv, wv, stream, zero_status);
  const long long M = static_cast<long long>(s->S) * s->T, C = static_cast<long long>(s->H) * 64;
  int rc = launch_linear_plain(x, w, b, qkv, M, 3 * C, C, wv.status, stream, zero_status);
  if (rc) return rc;
  return launch_prologue(mode, s, qkv, gq, bq, gk, bk, wv, stream, false);
}

int check_block_args(int mode, const vggt_attn_shape* s, const void* x, const void* w_qkv, const float* b_qkv,
                     const float* gq, const float* bq, const float* gk, const float* bk, const void* w_out,
                     const float* b_out, void* qkv, void* attn, void* y, void* ws, size_t ws_bytes) {
  int rc = check_prologue_args(mode, s, qkv, gq, bq, gk, bk, ws, ws_bytes);
  if (rc) return rc;
  if ((rc = check_core_args(mode, s, qkv, attn, ws, ws_bytes))) return rc;
  if (!x || !w_qkv || !w_out || !y) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_qkv, 16) || !aligned(w_out, 16) || !aligned(y, 16) ||
      (b_qkv && !aligned(b_qkv, 16)) || (b_out && !aligned(b_out, 16)))
    return VGGT_ATTN_ERR_MISALIGNED;
  const long long M = static_cast<long long>(s->S) * s->T, C = static_cast<long long>(s->H) * 64;
  if ((rc = check_linear_dims(M, 3 * C, C))) return rc;
  if (mode == VGGT_ATTN_REGISTER && 3LL * s->n_special > s->T) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  const size_t row = static_cast<size_t>(C) * 2;
  const size_t x_bytes = M * row, qkv_bytes = 3 * M * row;
  if (overlaps(y, x_bytes, attn, x_bytes) || overlaps(y, x_bytes, ws, ws_bytes) || overlaps(y, x_bytes, qkv, qkv_bytes) ||
      overlaps(y, x_bytes, x, x_bytes) || overlaps(qkv, qkv_bytes, x, x_bytes) || overlaps(attn, x_bytes, x, x_bytes) ||
      overlaps(ws, ws_bytes, x, x_bytes))
    return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

}  // namespace

extern "C" int vggt_attn_block(int mode, const vggt_attn_shape* shape, const void* x, const void* w_qkv,
                               const float* b_qkv, const float* q_gamma, const float* q_beta, const float* k_gamma,
                               const float* k_beta, const void* w_out, const float* b_out, void* qkv, void* attn,
                               void* y, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_block_args(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, w_out, b_out, qkv, attn, y,
                            workspace, workspace_bytes);
  if (rc) return rc;
  if ((rc = check_device())) return rc;
  const long long M = static_cast<long long>(shape->S) * shape->T, C = static_cast<long long>(shape->H) * 64;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (mode == VGGT_ATTN_REGISTER) {
    // Only the special tokens take part: gather their rows of x, run the block
    // on that compact sequence (register attention over it is global attention
    // without rotation), scatter the result rows back; patch rows of y are not
    // written.  Scratch: attn holds x_s, attn_s and y_s; qkv holds qkv_s.
    vggt_attn_shape s2 = *shape;
    s2.T = shape->n_special;
    s2.grid_h = 0;
    s2.grid_w = 0;
    const long long Ms = static_cast<long long>(shape->S) * shape->n_special;
    const size_t row = static_cast<size_t>(C) * 2;
    uint8_t* xs = static_cast<uint8_t*>(attn);
    uint8_t* as = xs + Ms * row;
    uint8_t* ys = as + Ms * row;
    const WorkspaceView wv = workspace_view(&s2, VGGT_ATTN_GLOBAL, workspace);
    if ((rc = launch_special_rows(x, xs, static_cast<int>(Ms), row, shape->n_special, shape->T, true, st))) return rc;
    if ((rc = launch_block_qkv(VGGT_ATTN_GLOBAL, &s2, xs, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, qkv, wv, st,
                               true)))
      return rc;
    if ((rc = launch_core(VGGT_ATTN_GLOBAL, &s2, qkv, as, wv, st))) return rc;
    if ((rc = launch_linear_plain(as, w_out, b_out, ys, Ms, C, C, wv.status, st))) return rc;
    return launch_special_rows(ys, y, static_cast<int>(Ms), row, shape->n_special, shape->T, false, st);
  }
  const WorkspaceView wv = workspace_view(shape, mode, workspace);
  if ((rc = launch_block_qkv(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, qkv, wv, st, true)))
    return rc;
  if ((rc = launch_core(mode, shape, qkv, attn, wv, st))) return rc;
  return launch_linear_plain(attn, w_out, b_out, y, M, C, C, wv.status, st);
}

// ---------------------------------------------------------------------------
// Subsampled global attention (AVGGT article, section B, point 2).
namespace {

struct SgaLayout {
  vggt::SgaGeometry g;
  WorkspaceView w;          // status, q plane, k plane (all tokens)
  uint16_t* ks;             // kept keys [H][Nk][64]
  uint16_t* vs;             // kept values [Nk][H][64]
  float* sums;              // [2][H][64]
  size_t bytes;
};

bool sga_layout(const vggt_attn_shape* s, int s_h, int s_w, void* ws, SgaLayout* out) {
  if (s_h < 1 || s_w < 1) return false;
  vggt::SgaGeometry g{};
  g.N = s->S * s->T;
  g.H = s->H;
  g.T = s->T;
  g.n_special = s->n_special;
  g.grid_w = s->grid_w > 0 ? s->grid_w : 1;
  g.s_h = s_h;
  g.s_w = s_w;
  g.grid_h = s->grid_h;
  const int nh = s->grid_h > 0 ? (s->grid_h + s_h - 1) / s_h : 0;
  g.nw = s->grid_w > 0 ? (s->grid_w + s_w - 1) / s_w : 0;
  g.kept_per_frame = s->n_special + nh * g.nw;
  g.Nk = s->S * g.kept_per_frame;
  if (g.Nk < 1) return false;
  SgaLayout L{};
  L.g = g;
  L.w = workspace_view(s, VGGT_ATTN_GLOBAL, ws);
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = L.w.bytes;
  const size_t ks_bytes = align256(static_cast<size_t>(g.Nk) * g.H * 64 * 2);
  L.ks = reinterpret_cast<uint16_t*>(base + off);
  off += ks_bytes;
  L.vs = reinterpret_cast<uint16_t*>(base + off);
  off += ks_bytes;
  L.sums = reinterpret_cast<float*>(base + off);
  off += align256(static_cast<size_t>(2) * g.H * 64 * 4);
  L.bytes = off;
  *out = L;
  return true;
}

}  // namespace

extern "C" size_t vggt_attn_sga_workspace_size(const vggt_attn_shape* shape, int s_h, int s_w) {
  if (check_shape(shape, VGGT_ATTN_GLOBAL) != VGGT_ATTN_OK) return 0;
  SgaLayout L;
  if (!sga_layout(shape, s_h, s_w, nullptr, &L)) return 0;
  return L.bytes;
}

extern "C" int vggt_attn_global_sga(const vggt_attn_shape* shape, int s_h, int s_w, const void* qkv,
                                    const float* q_gamma, const float* q_beta, const float* k_gamma,
                                    const float* k_beta, void* out, void* workspace, size_t workspace_bytes,
                                    void* cuda_stream) {
  int rc = check_shape(shape, VGGT_ATTN_GLOBAL);
  if (rc) return rc;
  if (s_h < 1 || s_w < 1 || s_h > 1024 || s_w > 1024) return VGGT_ATTN_ERR_INVALID_ARG;
  const size_t need = vggt_attn_sga_workspace_size(shape, s_h, s_w);
  if (need == 0) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (!workspace) return VGGT_ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < need) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  // The global-mode checks cover qkv, gamma/beta, out and their overlaps with
  // the part of the workspace they see; the rest is checked here.
  if ((rc = check_prologue_args(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace,
                                workspace_bytes)))
    return rc;
  if ((rc = check_core_args(VGGT_ATTN_GLOBAL, shape, qkv, out, workspace, workspace_bytes))) return rc;
  if ((rc = check_device())) return rc;
  SgaLayout L;
  sga_layout(shape, s_h, s_w, workspace, &L);
  const vggt::SgaGeometry& g = L.g;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // 1. QK-LayerNorm + RoPE of every token (global mode: one [N][64] plane per head).
  if ((rc = launch_prologue(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, L.w, st))) return rc;
  // 2. Sums over the discarded tokens, and the kept keys/values gathered.
  if (cudaMemsetAsync(L.sums, 0, static_cast<size_t>(2) * g.H * 64 * 4, st) != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return VGGT_ATTN_ERR_CUDA;
    const unsigned blocks = static_cast<unsigned>(std::max(1, std::min(g.N, sms * 8)));   // contiguous token ranges
    vggt::sga_sum_kernel<<<blocks, 256, 0, st>>>(g, L.w.k, static_cast<const uint16_t*>(qkv), L.sums);
    vggt::sga_gather_kernel<<<static_cast<unsigned>(std::min(g.Nk, sms * 16)), 256, 0, st>>>(
        g, L.w.k, static_cast<const uint16_t*>(qkv), L.ks, L.vs);
    if (cudaGetLastError() != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  }
  // 3. Attention of every query over the kept keys, plus the per-row diagonal
  //    and mean-pair terms in the epilogue.
  CUtensorMap mq, mk, mv;
  {
    const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};
    const cuuint32_t box_k[3] = {64, vggt::core::BN, 1};
    const cuuint64_t dq[3] = {64, static_cast<cuuint64_t>(g.N), static_cast<cuuint64_t>(g.H)};
    const cuuint64_t sq[2] = {128, static_cast<cuuint64_t>(g.N) * 128};
    const cuuint64_t dk[3] = {64, static_cast<cuuint64_t>(g.Nk), static_cast<cuuint64_t>(g.H)};
    const cuuint64_t sk[2] = {128, static_cast<cuuint64_t>(g.Nk) * 128};
    if (!make_map(&mq, L.w.q, 3, dq, sq, box_q) || !make_map(&mk, L.ks, 3, dk, sk, box_k)) return VGGT_ATTN_ERR_CUDA;
    const cuuint32_t box_v[4] = {64, 1, vggt::core::BN, 1};
    const cuuint64_t dv[4] = {64, static_cast<cuuint64_t>(g.H), static_cast<cuuint64_t>(g.Nk), 1};
    const cuuint64_t sv[3] = {128, static_cast<cuuint64_t>(g.H) * 128, static_cast<cuuint64_t>(g.Nk) * g.H * 128};
    if (!make_map(&mv, L.vs, 4, dv, sv, box_v)) return VGGT_ATTN_ERR_CUDA;
  }
  vggt::CoreParams p{};
  p.L = g.N;
  p.Lk = g.Nk;
  p.H = g.H;
  p.B = 1;
  p.out_T = shape->T;
  p.out_group = g.N;
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = static_cast<long long>(g.N) * g.H * 64;
  p.status = L.w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  const int n_d = g.N - g.Nk;
  p.sga = {L.w.q, L.w.k, static_cast<const uint16_t*>(qkv), L.sums, n_d, n_d > 0 ? 1.0f / n_d : 0.0f,
           g.T, g.n_special, g.grid_w, g.s_h, g.s_w};
  ModeGeometry mg{1, g.N, g.N, 2};
  return launch_core_cfg<vggt::CoreCfg<2, true>>(mg, g.H, mq, mk, mv, p, st);
}

// ---------------------------------------------------------------------------
// Descriptor attention (FlashVGGT article, abstract): every query over the
// per-frame descriptors (special tokens, window means of the patch grid).
extern "C" int vggt_attn_global_desc(const vggt_attn_shape* shape, int s_h, int s_w, const void* qkv,
                                     const float* q_gamma, const float* q_beta, const float* k_gamma,
                                     const float* k_beta, void* out, void* workspace, size_t workspace_bytes,
                                     void* cuda_stream) {
  int rc = check_shape(shape, VGGT_ATTN_GLOBAL);
  if (rc) return rc;
  if (s_h < 1 || s_w < 1 || s_h > 1024 || s_w > 1024) return VGGT_ATTN_ERR_INVALID_ARG;
  const size_t need = vggt_attn_sga_workspace_size(shape, s_h, s_w);   // same layout: descriptors in place of kept keys
  if (need == 0) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (!workspace) return VGGT_ATTN_ERR_INVALID_ARG;
  if (workspace_bytes < need) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  if ((rc = check_prologue_args(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace,
                                workspace_bytes)))
    return rc;
  if ((rc = check_core_args(VGGT_ATTN_GLOBAL, shape, qkv, out, workspace, workspace_bytes))) return rc;
  if ((rc = check_device())) return rc;
  SgaLayout L;
  sga_layout(shape, s_h, s_w, workspace, &L);
  const vggt::SgaGeometry& g = L.g;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  // 1. QK-LayerNorm + RoPE of every token; 2. the descriptors (window means).
  if ((rc = launch_prologue(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, L.w, st))) return rc;
  {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
      return VGGT_ATTN_ERR_CUDA;
    vggt::desc_pool_kernel<<<static_cast<unsigned>(std::min(g.Nk, sms * 16)), 256, 0, st>>>(
        g, L.w.k, static_cast<const uint16_t*>(qkv), L.ks, L.vs);
    if (cudaGetLastError() != cudaSuccess) return VGGT_ATTN_ERR_CUDA;
  }
  // 3. Plain attention of every query over the descriptors.
  CUtensorMap mq, mk, mv;
  {
    const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};
    const cuuint32_t box_k[3] = {64, vggt::core::BN, 1};
    const cuuint64_t dq[3] = {64, static_cast<cuuint64_t>(g.N), static_cast<cuuint64_t>(g.H)};
    const cuuint64_t sq[2] = {128, static_cast<cuuint64_t>(g.N) * 128};
    const cuuint64_t dk[3] = {64, static_cast<cuuint64_t>(g.Nk), static_cast<cuuint64_t>(g.H)};
    const cuuint64_t sk[2] = {128, static_cast<cuuint64_t>(g.Nk) * 128};
    if (!make_map(&mq, L.w.q, 3, dq, sq, box_q) || !make_map(&mk, L.ks, 3, dk, sk, box_k)) return VGGT_ATTN_ERR_CUDA;
    const cuuint32_t box_v[4] = {64, 1, vggt::core::BN, 1};
    const cuuint64_t dv[4] = {64, static_cast<cuuint64_t>(g.H), static_cast<cuuint64_t>(g.Nk), 1};
    const cuuint64_t sv[3] = {128, static_cast<cuuint64_t>(g.H) * 128, static_cast<cuuint64_t>(g.Nk) * g.H * 128};
    if (!make_map(&mv, L.vs, 4, dv, sv, box_v)) return VGGT_ATTN_ERR_CUDA;
  }
  vggt::CoreParams p{};
  p.L = g.N;
  p.Lk = g.Nk;
  p.H = g.H;
  p.B = 1;
  p.out_T = shape->T;
  p.out_group = g.N;
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = static_cast<long long>(g.N) * g.H * 64;
  p.status = L.w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  ModeGeometry mg{1, g.N, g.N, 2};
  return launch_core_cfg<vggt::CoreCfg<2>>(mg, g.H, mq, mk, mv, p, st);
}

// ---------------------------------------------------------------------------
// Transformer blocks and the alternating-attention schedule (VGGT-Omega
// Aggregator explainer, section 3).
namespace {

constexpr int kMaxBlockChannels = 2048;   // LayerNorm kernel: up to 8 16-byte chunks per lane

struct BlockLayout {
  vggt_attn_shape s;        // the shape the block's kernels see (register mode: special tokens only)
  int mode;                 // the attention mode they run (register mode: global)
  long long M;              // rows the block processes
  WorkspaceView att;        // attention workspace (status word first)
  uint8_t* xs;              // register mode: the gathered rows of x [M][C]
  uint8_t* h;               // norm output [M][C]
  uint8_t* big;             // qkv [M][3C] then attention output [M][C]; later the hidden [M][4C]
  size_t bytes;
};

BlockLayout block_layout(const vggt_attn_shape* shape, int mode, void* ws) {
  BlockLayout L{};
  L.s = *shape;
  L.mode = mode;
  if (mode == VGGT_ATTN_REGISTER) {
    L.s.T = shape->n_special;
    L.s.grid_h = 0;
    L.s.grid_w = 0;
    L.mode = VGGT_ATTN_GLOBAL;
  }
  L.M = static_cast<long long>(L.s.S) * L.s.T;
  const size_t row = static_cast<size_t>(shape->H) * 64 * 2;
  L.att = workspace_view(&L.s, L.mode, ws);
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = L.att.bytes;
  if (mode == VGGT_ATTN_REGISTER) {
    L.xs = base + off;
    off += align256(L.M * row);
  }
  L.h = base + off;
  off += align256(L.M * row);
  L.big = base + off;
  off += align256(L.M * 4 * row);
  L.bytes = off;
  return L;
}

int check_block_shape(const vggt_attn_shape* s, int mode) {
  int rc = check_shape(s, mode);
  if (rc) return rc;
  const long long C = static_cast<long long>(s->H) * 64;
  if (C % 256 || C > kMaxBlockChannels) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  const long long M = static_cast<long long>(s->S) * (mode == VGGT_ATTN_REGISTER ? s->n_special : s->T);
  if ((rc = check_linear_dims(M, 4 * C, C)) || (rc = check_linear_dims(M, C, 4 * C))) return rc;
  return VGGT_ATTN_OK;
}

bool vec_ok(const float* p, bool optional) { return p ? aligned(p, 16) : optional; }

int check_block_weights(const vggt_block_weights* w, long long C, const void* x, size_t x_bytes, const void* ws,
                        size_t ws_bytes) {
  if (!w) return VGGT_ATTN_ERR_INVALID_ARG;
  const float* req[] = {w->norm1_gamma, w->norm1_beta, w->q_gamma, w->q_beta, w->k_gamma,
                        w->k_beta,      w->ls1,        w->norm2_gamma, w->norm2_beta, w->ls2};
  for (const float* v : req)
    if (!v) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!w->w_qkv || !w->w_proj || !w->w_fc1 || !w->w_fc2) return VGGT_ATTN_ERR_INVALID_ARG;
  for (const float* v : req)
    if (!vec_ok(v, false)) return VGGT_ATTN_ERR_MISALIGNED;
  if (!vec_ok(w->b_qkv, true) || !vec_ok(w->b_proj, true) || !vec_ok(w->b_fc1, true) || !vec_ok(w->b_fc2, true))
    return VGGT_ATTN_ERR_MISALIGNED;
  if (!aligned(w->w_qkv, 16) || !aligned(w->w_proj, 16) || !aligned(w->w_fc1, 16) || !aligned(w->w_fc2, 16))
    return VGGT_ATTN_ERR_MISALIGNED;
  const size_t cc = static_cast<size_t>(C) * C * 2;
  const void* mats[4] = {w->w_qkv, w->w_proj, w->w_fc1, w->w_fc2};
  const size_t mat_bytes[4] = {3 * cc, cc, 4 * cc, 4 * cc};
  for (int i = 0; i < 4; ++i)
    if (overlaps(x, x_bytes, mats[i], mat_bytes[i]) || overlaps(ws, ws_bytes, mats[i], mat_bytes[i]))
      return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

int launch_layernorm(const void* x, void* y, const float* gamma, const float* beta, long long M, long long C,
                     float eps, int* status, bool zero_status, cudaStream_t st) {
  vggt::LayerNormParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.y = static_cast<uint16_t*>(y);
  p.gamma = gamma;
  p.beta = beta;
  p.M = M;
  p.eps = eps;
  p.status = status;
  p.zero_status = zero_status ? 1 : 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return VGGT_ATTN_ERR_CUDA;
  long long blocks = (M + 7) / 8;                    // 8 rows (warps) per block
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  const unsigned grid = static_cast<unsigned>(blocks);
  switch (C / 256) {
    case 1: vggt::layernorm_rows_kernel<1><<<grid, 256, 0, st>>>(p); break;
    case 2: vggt::layernorm_rows_kernel<2><<<grid, 256, 0, st>>>(p); break;
    case 3: vggt::layernorm_rows_kernel<3><<<grid, 256, 0, st>>>(p); break;
    case 4: vggt::layernorm_rows_kernel<4><<<grid, 256, 0, st>>>(p); break;
    case 5: vggt::layernorm_rows_kernel<5><<<grid, 256, 0, st>>>(p); break;
    case 6: vggt::layernorm_rows_kernel<6><<<grid, 256, 0, st>>>(p); break;
    case 7: vggt::layernorm_rows_kernel<7><<<grid, 256, 0, st>>>(p); break;
    case 8: vggt::layernorm_rows_kernel<8><<<grid, 256, 0, st>>>(p); break;
    default: return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  }
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

// The kernels of one block; arguments already validated.
// clear_status: this block's first kernel clears the status word (the first
// block of a call); later blocks keep what earlier ones recorded.
int run_block(int mode, const vggt_attn_shape* shape, void* x, const vggt_block_weights* w, float eps, void* ws,
              bool clear_status, cudaStream_t st) {
  const BlockLayout L = block_layout(shape, mode, ws);
  const long long C = static_cast<long long>(shape->H) * 64, M = L.M;
  int* status = L.att.status;
  int rc;
  void* xb = x;
  if (mode == VGGT_ATTN_REGISTER) {
    if ((rc = launch_special_rows(x, L.xs, static_cast<int>(M), C * 2, shape->n_special, shape->T, true, st)))
      return rc;
    xb = L.xs;
  }
  uint8_t* qkv = L.big;
  uint8_t* att = L.big + static_cast<size_t>(M) * 3 * C * 2;
  if ((rc = launch_layernorm(xb, L.h, w->norm1_gamma, w->norm1_beta, M, C, eps, status, clear_status, st)))
    return rc;
  if ((rc = launch_block_qkv(L.mode, &L.s, L.h, w->w_qkv, w->b_qkv, w->q_gamma, w->q_beta, w->k_gamma, w->k_beta, qkv,
                              L.att, st, false)))
    return rc;
  if ((rc = launch_core(L.mode, &L.s, qkv, att, L.att, st))) return rc;
  if ((rc = launch_linear_plain(att, w->w_proj, w->b_proj, xb, M, C, C, status, st, false, vggt::lin::EPI_RESID, xb,
                                w->ls1)))
    return rc;
  if ((rc = launch_layernorm(xb, L.h, w->norm2_gamma, w->norm2_beta, M, C, eps, status, false, st))) return rc;
  if ((rc = launch_linear_plain(L.h, w->w_fc1, w->b_fc1, L.big, M, 4 * C, C, status, st, false, vggt::lin::EPI_GELU)))
    return rc;
  if ((rc = launch_linear_plain(L.big, w->w_fc2, w->b_fc2, xb, M, C, 4 * C, status, st, false, vggt::lin::EPI_RESID,
                                xb, w->ls2)))
    return rc;
  if (mode == VGGT_ATTN_REGISTER)
    return launch_special_rows(L.xs, x, static_cast<int>(M), C * 2, shape->n_special, shape->T, false, st);
  return VGGT_ATTN_OK;
}

int check_block_common(const vggt_attn_shape* shape, void* x, void* ws, size_t ws_bytes, size_t need) {
  if (!x || !ws) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(ws, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  if (ws_bytes < need) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  const size_t x_bytes = static_cast<size_t>(shape->S) * shape->T * shape->H * 64 * 2;
  if (overlaps(x, x_bytes, ws, ws_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  return VGGT_ATTN_OK;
}

}  // namespace

extern "C" size_t vggt_block_workspace_size(const vggt_attn_shape* shape, int mode) {
  if (check_block_shape(shape, mode) != VGGT_ATTN_OK) return 0;
  return block_layout(shape, mode, nullptr).bytes;
}

extern "C" int vggt_block_forward(int mode, const vggt_attn_shape* shape, void* x, const vggt_block_weights* w,
                                  float norm_eps, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_block_shape(shape, mode);
  if (rc) return rc;
  if (!std::isfinite(norm_eps) || !(norm_eps > 0.f)) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_block_common(shape, x, workspace, workspace_bytes, vggt_block_workspace_size(shape, mode))))
    return rc;
  const size_t x_bytes = static_cast<size_t>(shape->S) * shape->T * shape->H * 64 * 2;
  if ((rc = check_block_weights(w, static_cast<long long>(shape->H) * 64, x, x_bytes, workspace, workspace_bytes)))
    return rc;
  if ((rc = check_device())) return rc;
  return run_block(mode, shape, x, w, norm_eps, workspace, true, static_cast<cudaStream_t>(cuda_stream));
}

extern "C" size_t vggt_aggregator_workspace_size(const vggt_attn_shape* shape) {
  size_t need = 0;
  for (int mode : {VGGT_ATTN_FRAME, VGGT_ATTN_GLOBAL, VGGT_ATTN_REGISTER}) {
    if (mode == VGGT_ATTN_REGISTER && (!shape || shape->n_special < 1)) continue;
    const size_t b = vggt_block_workspace_size(shape, mode);
    if (b == 0) return 0;
    need = std::max(need, b);
  }
  return need;
}

extern "C" int vggt_aggregator_forward_cached(const vggt_attn_shape* shape, void* x,
                                              const vggt_block_weights* frame_blocks,
                                              const vggt_block_weights* inter_blocks, int n_layers,
                                              const int* register_layers, int n_register, const int* cache_layers,
                                              int n_cache, void* const* cache_out, float norm_eps, void* workspace,
                                              size_t workspace_bytes, void* cuda_stream) {
  if (n_layers < 0 || n_register < 0 || (n_register > 0 && !register_layers)) return VGGT_ATTN_ERR_INVALID_ARG;
  if (n_cache < 0 || (n_cache > 0 && (!cache_layers || !cache_out))) return VGGT_ATTN_ERR_INVALID_ARG;
  if (n_layers > 0 && (!frame_blocks || !inter_blocks)) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(norm_eps) || !(norm_eps > 0.f)) return VGGT_ATTN_ERR_INVALID_ARG;
  int rc;
  if ((rc = check_block_shape(shape, VGGT_ATTN_FRAME)) || (rc = check_block_shape(shape, VGGT_ATTN_GLOBAL)))
    return rc;
  for (int i = 0; i < n_register; ++i)
    if (register_layers[i] < 0 || register_layers[i] >= n_layers) return VGGT_ATTN_ERR_INVALID_ARG;
  if (n_register > 0 && (rc = check_block_shape(shape, VGGT_ATTN_REGISTER))) return rc;
  if ((rc = check_block_common(shape, x, workspace, workspace_bytes, vggt_aggregator_workspace_size(shape))))
    return rc;
  const long long C = static_cast<long long>(shape->H) * 64;
  const size_t x_bytes = static_cast<size_t>(shape->S) * shape->T * C * 2;
  for (int l = 0; l < n_layers; ++l)
    if ((rc = check_block_weights(&frame_blocks[l], C, x, x_bytes, workspace, workspace_bytes)) ||
        (rc = check_block_weights(&inter_blocks[l], C, x, x_bytes, workspace, workspace_bytes)))
      return rc;
  for (int i = 0; i < n_cache; ++i) {
    if (cache_layers[i] < 0 || cache_layers[i] >= n_layers || !cache_out[i]) return VGGT_ATTN_ERR_INVALID_ARG;
    if (!aligned(cache_out[i], 16)) return VGGT_ATTN_ERR_MISALIGNED;
    if (overlaps(cache_out[i], 2 * x_bytes, x, x_bytes) || overlaps(cache_out[i], 2 * x_bytes, workspace, workspace_bytes))
      return VGGT_ATTN_ERR_INVALID_ARG;
  }
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const size_t row = static_cast<size_t>(C) * 2;
  const size_t rows = static_cast<size_t>(shape->S) * shape->T;
  // x into channels [half*C, (half+1)*C) of every cache buffer kept for layer l.
  auto cache = [&](int l, int half) -> int {
    for (int i = 0; i < n_cache; ++i)
      if (cache_layers[i] == l &&
          cudaMemcpy2DAsync(static_cast<uint8_t*>(cache_out[i]) + half * row, 2 * row, x, row, row, rows,
                            cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return VGGT_ATTN_ERR_CUDA;
    return VGGT_ATTN_OK;
  };
  for (int l = 0; l < n_layers; ++l) {
    bool reg = false;
    for (int i = 0; i < n_register; ++i) reg = reg || register_layers[i] == l;
    if ((rc = run_block(VGGT_ATTN_FRAME, shape, x, &frame_blocks[l], norm_eps, workspace, l == 0, st))) return rc;
    if ((rc = cache(l, 0))) return rc;
    if ((rc = run_block(reg ? VGGT_ATTN_REGISTER : VGGT_ATTN_GLOBAL, shape, x, &inter_blocks[l], norm_eps, workspace,
                        false, st)))
      return rc;
    if ((rc = cache(l, 1))) return rc;
  }
  return VGGT_ATTN_OK;
}

extern "C" int vggt_aggregator_forward(const vggt_attn_shape* shape, void* x, const vggt_block_weights* frame_blocks,
                                       const vggt_block_weights* inter_blocks, int n_layers,
                                       const int* register_layers, int n_register, float norm_eps, void* workspace,
                                       size_t workspace_bytes, void* cuda_stream) {
  return vggt_aggregator_forward_cached(shape, x, frame_blocks, inter_blocks, n_layers, register_layers, n_register,
                                        nullptr, 0, nullptr, norm_eps, workspace, workspace_bytes, cuda_stream);
}

// ---------------------------------------------------------------------------
// Camera-head trunk (VGGT-Omega Aggregator explainer, section 4).
namespace {

vggt_attn_shape camera_trunk_shape(const vggt_attn_shape* s) {
  vggt_attn_shape c = *s;
  c.T = s->n_special;
  c.grid_h = 0;
  c.grid_w = 0;
  return c;
}

}  // namespace

extern "C" size_t vggt_camera_trunk_workspace_size(const vggt_attn_shape* shape) {
  if (!shape || shape->n_special < 1 || check_shape(shape, VGGT_ATTN_REGISTER) != VGGT_ATTN_OK) return 0;
  const vggt_attn_shape c = camera_trunk_shape(shape);
  return vggt_block_workspace_size(&c, VGGT_ATTN_GLOBAL);
}

extern "C" int vggt_camera_trunk_forward(const vggt_attn_shape* shape, const void* feats, void* tokens,
                                         const vggt_block_weights* blocks, int n_blocks, float norm_eps,
                                         void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_shape(shape, VGGT_ATTN_REGISTER);
  if (rc) return rc;
  if (n_blocks < 0 || (n_blocks > 0 && !blocks) || !feats) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(norm_eps) || !(norm_eps > 0.f)) return VGGT_ATTN_ERR_INVALID_ARG;
  const vggt_attn_shape c = camera_trunk_shape(shape);
  if ((rc = check_block_shape(&c, VGGT_ATTN_GLOBAL))) return rc;
  if (!aligned(feats, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  if ((rc = check_block_common(&c, tokens, workspace, workspace_bytes, vggt_camera_trunk_workspace_size(shape))))
    return rc;
  const long long C = static_cast<long long>(shape->H) * 64;
  const size_t feats_bytes = static_cast<size_t>(shape->S) * shape->T * C * 2;
  const size_t tok_bytes = static_cast<size_t>(c.S) * c.T * C * 2;
  if (overlaps(feats, feats_bytes, tokens, tok_bytes) || overlaps(feats, feats_bytes, workspace, workspace_bytes))
    return VGGT_ATTN_ERR_INVALID_ARG;
  for (int b = 0; b < n_blocks; ++b)
    if ((rc = check_block_weights(&blocks[b], C, tokens, tok_bytes, workspace, workspace_bytes))) return rc;
  if ((rc = check_device())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const long long rows = static_cast<long long>(c.S) * c.T;
  if ((rc = launch_special_rows(feats, tokens, static_cast<int>(rows), C * 2, shape->n_special, shape->T, true, st)))
    return rc;
  for (int b = 0; b < n_blocks; ++b)
    if ((rc = run_block(VGGT_ATTN_GLOBAL, &c, tokens, &blocks[b], norm_eps, workspace, b == 0, st))) return rc;
  return VGGT_ATTN_OK;
}

// ---------------------------------------------------------------------------
// Query-sharded global attention: local prologue, all-gather of k and v by
// the caller, core over all ranks' keys.
namespace {

constexpr int kMaxShardWorld = 1024;

struct ShardLayout {
  WorkspaceView w;          // status, q plane [H][L][64] (k plane unused)
  uint16_t* k_send;         // [L][H][64]
  uint16_t* v_send;
  uint16_t* k_all;          // [world L][H][64]
  uint16_t* v_all;
  float* part_o;            // [H][L][64]: softmax state over the rank's own keys (overlapped form)
  float* part_ml;           // [H][L][2]
  long long L, Lk;
  size_t bytes;
};

ShardLayout shard_layout(const vggt_attn_shape* s, int world, void* ws) {
  ShardLayout S{};
  S.L = static_cast<long long>(s->S) * s->T;
  S.Lk = S.L * world;
  const size_t row = static_cast<size_t>(s->H) * 64 * 2;
  uint8_t* base = static_cast<uint8_t*>(ws);
  S.w.status = reinterpret_cast<int*>(base);
  size_t off = kStatusBytes;
  S.w.q = reinterpret_cast<uint16_t*>(base + off);
  off += align256(S.L * row);
  S.w.k = nullptr;
  S.w.v = nullptr;
  S.k_send = reinterpret_cast<uint16_t*>(base + off);
  off += align256(S.L * row);
  S.v_send = reinterpret_cast<uint16_t*>(base + off);
  off += align256(S.L * row);
  S.k_all = reinterpret_cast<uint16_t*>(base + off);
  off += align256(S.Lk * row);
  S.v_all = reinterpret_cast<uint16_t*>(base + off);
  off += align256(S.Lk * row);
  S.part_o = reinterpret_cast<float*>(base + off);
  off += align256(static_cast<size_t>(s->H) * S.L * 64 * sizeof(float));
  S.part_ml = reinterpret_cast<float*>(base + off);
  off += align256(static_cast<size_t>(s->H) * S.L * 2 * sizeof(float));
  S.w.bytes = off;
  S.bytes = off;
  return S;
}

int check_shard_shape(const vggt_attn_shape* s, int world) {
  if (world < 1 || world > kMaxShardWorld) return VGGT_ATTN_ERR_INVALID_ARG;
  int rc = check_shape(s, VGGT_ATTN_GLOBAL);
  if (rc) return rc;
  vggt_attn_shape whole = *s;
  const long long S = static_cast<long long>(s->S) * world;
  if (S > INT32_MAX) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  whole.S = static_cast<int>(S);
  return check_shape(&whole, VGGT_ATTN_GLOBAL);   // token counts of the whole scene
}

// fused_prefix: only the status word, q plane and send buffers are needed (the
// prologue, and the core that reads every rank's send buffers in place).
int check_shard_ws(const vggt_attn_shape* s, int world, void* ws, size_t ws_bytes, bool fused_prefix = false) {
  if (!ws) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  const ShardLayout L = shard_layout(s, world, nullptr);
  const size_t need = fused_prefix ? static_cast<size_t>(reinterpret_cast<uintptr_t>(L.k_all)) : L.bytes;
  if (ws_bytes < need) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  return VGGT_ATTN_OK;
}

}  // namespace

extern "C" size_t vggt_attn_shard_workspace_size(const vggt_attn_shape* shape, int world) {
  if (check_shard_shape(shape, world) != VGGT_ATTN_OK) return 0;
  return shard_layout(shape, world, nullptr).bytes;
}

extern "C" int vggt_attn_shard_buffers(const vggt_attn_shape* shape, int world, void* workspace, void** k_send,
                                       void** v_send, void** k_all, void** v_all) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if (!workspace || !k_send || !v_send || !k_all || !v_all) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return VGGT_ATTN_ERR_MISALIGNED;
  const ShardLayout L = shard_layout(shape, world, workspace);
  *k_send = L.k_send;
  *v_send = L.v_send;
  *k_all = L.k_all;
  *v_all = L.v_all;
  return VGGT_ATTN_OK;
}

extern "C" int vggt_attn_global_shard_prologue(const vggt_attn_shape* shape, int world, const void* qkv,
                                               const float* q_gamma, const float* q_beta, const float* k_gamma,
                                               const float* k_beta, void* workspace, size_t workspace_bytes,
                                               void* cuda_stream) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if ((rc = check_shard_ws(shape, world, workspace, workspace_bytes, true))) return rc;
  if (!qkv || !q_gamma || !q_beta || !k_gamma || !k_beta) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(qkv, 16) || !aligned(q_gamma, 16) || !aligned(q_beta, 16) || !aligned(k_gamma, 16) ||
      !aligned(k_beta, 16))
    return VGGT_ATTN_ERR_MISALIGNED;
  const size_t qkv_bytes = static_cast<size_t>(shape->S) * shape->T * 3 * shape->H * 128;
  if (overlaps(qkv, qkv_bytes, workspace, workspace_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  const ShardLayout L = shard_layout(shape, world, workspace);
  return launch_prologue(VGGT_ATTN_GLOBAL, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, L.w,
                         static_cast<cudaStream_t>(cuda_stream), true, L.k_send, L.v_send);
}

extern "C" int vggt_attn_global_shard_core(const vggt_attn_shape* shape, int world, void* out, void* workspace,
                                           size_t workspace_bytes, void* cuda_stream) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if ((rc = check_shard_ws(shape, world, workspace, workspace_bytes))) return rc;
  if (!out) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  const size_t out_bytes = static_cast<size_t>(shape->S) * shape->T * shape->H * 128;
  if (overlaps(out, out_bytes, workspace, workspace_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  const ShardLayout L = shard_layout(shape, world, workspace);
  const long long H = shape->H;
  CUtensorMap mq, mk, mv;
  {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(L.L), static_cast<cuuint64_t>(H)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(L.L) * 128};
    const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};
    if (!make_map(&mq, L.w.q, 3, dims, strides, box_q)) return VGGT_ATTN_ERR_CUDA;
  }
  {
    // gathered keys and values, [Lk][H][64]: (dim, head, token, 1)
    const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L.Lk), 1};
    const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(L.Lk) * H * 128};
    const cuuint32_t box[4] = {64, 1, vggt::core::BN, 1};
    if (!make_map(&mk, L.k_all, 4, dims, strides, box) || !make_map(&mv, L.v_all, 4, dims, strides, box))
      return VGGT_ATTN_ERR_CUDA;
  }
  vggt::CoreParams p{};
  p.L = static_cast<int>(L.L);
  p.Lk = static_cast<int>(L.Lk);
  p.H = shape->H;
  p.B = 1;
  p.out_T = shape->T;
  p.out_group = static_cast<int>(L.L);
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = static_cast<long long>(shape->S) * shape->T * shape->H * 64;
  p.status = L.w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  ModeGeometry g{1, L.L, L.L, 2};
  return launch_core_cfg<vggt::CoreCfg<2, false, true>>(g, shape->H, mq, mk, mv, p, static_cast<cudaStream_t>(cuda_stream));
}

// Overlapped form: the rank's own keys first (from its send buffers, while the
// all-gather runs), then the other ranks' blocks of the gathered buffers with
// the first launch's softmax state merged in the epilogue.
namespace {

bool shard_q_map(CUtensorMap* mq, const ShardLayout& L, long long H) {
  const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(L.L), static_cast<cuuint64_t>(H)};
  const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(L.L) * 128};
  const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};
  return make_map(mq, L.w.q, 3, dims, strides, box_q);
}

// keys or values of one rank, [L][H][64] as (dim, head, token, 1); rows past L read as zeros
bool shard_block_map(CUtensorMap* m, const void* base, const ShardLayout& L, long long H) {
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L.L), 1};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(L.L) * H * 128};
  const cuuint32_t box[4] = {64, 1, vggt::core::BN, 1};
  return make_map(m, base, 4, dims, strides, box);
}

vggt::CoreParams shard_core_params(const vggt_attn_shape* shape, const ShardLayout& L, void* out) {
  vggt::CoreParams p{};
  p.L = static_cast<int>(L.L);
  p.H = shape->H;
  p.B = 1;
  p.out_T = shape->T;
  p.out_group = static_cast<int>(L.L);
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = out ? static_cast<long long>(shape->S) * shape->T * shape->H * 64 : 0;
  p.status = L.w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.part_o = L.part_o;
  p.part_ml = L.part_ml;
  p.part_rows = static_cast<long long>(shape->H) * L.L;
  return p;
}

}  // namespace

extern "C" int vggt_attn_global_shard_core_local(const vggt_attn_shape* shape, int world, void* workspace,
                                                 size_t workspace_bytes, void* cuda_stream) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if ((rc = check_shard_ws(shape, world, workspace, workspace_bytes))) return rc;
  if ((rc = check_device())) return rc;
  const ShardLayout L = shard_layout(shape, world, workspace);
  CUtensorMap mq, mk, mv;
  if (!shard_q_map(&mq, L, shape->H) || !shard_block_map(&mk, L.k_send, L, shape->H) ||
      !shard_block_map(&mv, L.v_send, L, shape->H))
    return VGGT_ATTN_ERR_CUDA;
  vggt::CoreParams p = shard_core_params(shape, L, nullptr);
  p.Lk = static_cast<int>(L.L);
  ModeGeometry g{1, L.L, L.L, 2};
  return launch_core_cfg<vggt::CoreCfg<2, false, true, false, 1>>(g, shape->H, mq, mk, mv, p,
                                                                  static_cast<cudaStream_t>(cuda_stream));
}

extern "C" int vggt_attn_global_shard_core_remote(const vggt_attn_shape* shape, int world, int rank, void* out,
                                                  void* workspace, size_t workspace_bytes, void* cuda_stream) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if (world < 2 || world - 1 > vggt::kMaxRankMaps) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if (rank < 0 || rank >= world) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_shard_ws(shape, world, workspace, workspace_bytes))) return rc;
  if (!out) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  const size_t out_bytes = static_cast<size_t>(shape->S) * shape->T * shape->H * 128;
  if (overlaps(out, out_bytes, workspace, workspace_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  using C = vggt::CoreCfg<2, false, true, true, 2>;
  const ShardLayout L = shard_layout(shape, world, workspace);
  const long long H = shape->H;
  CUtensorMap mq;
  if (!shard_q_map(&mq, L, H)) return VGGT_ATTN_ERR_CUDA;
  vggt::RankMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const size_t block = static_cast<size_t>(L.L) * H * 64;   // elements of one rank's block
  for (int q = 0, n = 0; q < world; ++q) {
    if (q == rank) continue;
    if (!shard_block_map(&maps.k[n], L.k_all + q * block, L, H) ||
        !shard_block_map(&maps.v[n], L.v_all + q * block, L, H))
      return VGGT_ATTN_ERR_CUDA;
    ++n;
  }
  const int spr = static_cast<int>((L.L + vggt::core::BN - 1) / vggt::core::BN);
  vggt::CoreParams p = shard_core_params(shape, L, out);
  p.Lk = (world - 1) * spr * vggt::core::BN;   // n_kv = (world - 1) * spr steps
  p.rank_tokens = static_cast<int>(L.L);
  p.rank_steps = spr;
  if (cudaFuncSetAttribute(vggt::attn_core_ranks_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_ALLOC) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  cudaFuncAttributes fa;   // the register split assumes the compiled count (see launch_core_cfg)
  if (cudaFuncGetAttributes(&fa, vggt::attn_core_ranks_kernel<C>) != cudaSuccess || fa.numRegs < C::REGS_AT_LAUNCH)
    return VGGT_ATTN_ERR_CUDA;
  const long long n_q = (L.L + 2 * vggt::core::BM - 1) / (2 * vggt::core::BM);
  const dim3 grid(static_cast<unsigned>(n_q), static_cast<unsigned>(H), 1);
  vggt::attn_core_ranks_kernel<C><<<grid, C::THREADS, C::SMEM_ALLOC, static_cast<cudaStream_t>(cuda_stream)>>>(
      mq, maps, p);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Host-memory pipeline: copies of neighbouring items overlap each item's kernels.
namespace {

struct PipeLayout {
  size_t att_bytes, qkv_bytes, out_bytes, bytes;
  uint8_t* qkv[2];
  uint8_t* out[2];
};

PipeLayout pipe_layout(const vggt_attn_shape* s, int mode, void* ws) {
  PipeLayout P{};
  P.att_bytes = workspace_view(s, mode, nullptr).bytes;
  P.qkv_bytes = static_cast<size_t>(s->S) * s->T * 3 * s->H * 128;
  P.out_bytes = static_cast<size_t>(s->S) * s->T * s->H * 128;
  uint8_t* base = static_cast<uint8_t*>(ws);
  size_t off = align256(P.att_bytes);
  for (int b = 0; b < 2; ++b) {
    P.qkv[b] = base + off;
    off += align256(P.qkv_bytes);
  }
  for (int b = 0; b < 2; ++b) {
    P.out[b] = base + off;
    off += align256(P.out_bytes);
  }
  P.bytes = off;
  return P;
}

bool pinned_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();   // clear the query's error state
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

}  // namespace

extern "C" size_t vggt_attn_host_pipeline_workspace_size(const vggt_attn_shape* shape, int mode) {
  if (check_shape(shape, mode) != VGGT_ATTN_OK) return 0;
  return pipe_layout(shape, mode, nullptr).bytes;
}

extern "C" int vggt_attn_host_pipeline(int mode, const vggt_attn_shape* shape, int n_items, const void* const* h_qkv,
                                       const float* q_gamma, const float* q_beta, const float* k_gamma,
                                       const float* k_beta, void* const* h_out, void* workspace,
                                       size_t workspace_bytes, void* compute_stream, void* h2d_stream,
                                       void* d2h_stream) {
  int rc = check_shape(shape, mode);
  if (rc) return rc;
  if (n_items < 0 || (n_items > 0 && (!h_qkv || !h_out)) || !workspace) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!q_gamma || !q_beta || !k_gamma || !k_beta) return VGGT_ATTN_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(q_gamma, 16) || !aligned(q_beta, 16) || !aligned(k_gamma, 16) ||
      !aligned(k_beta, 16))
    return VGGT_ATTN_ERR_MISALIGNED;
  const PipeLayout P = pipe_layout(shape, mode, workspace);
  if (workspace_bytes < P.bytes) return VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL;
  for (int i = 0; i < n_items; ++i)
    if (!h_qkv[i] || !h_out[i]) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  for (int i = 0; i < n_items; ++i)
    if (!pinned_host(h_qkv[i]) || !pinned_host(h_out[i])) return VGGT_ATTN_ERR_INVALID_ARG;
  if (n_items == 0) return VGGT_ATTN_OK;
  cudaStream_t sc = static_cast<cudaStream_t>(compute_stream);
  cudaStream_t si = static_cast<cudaStream_t>(h2d_stream);
  cudaStream_t so = static_cast<cudaStream_t>(d2h_stream);
  cudaEvent_t ev[3][2] = {};   // [h2d done, compute done, d2h done][staging set]
  for (int k = 0; k < 3 && rc == VGGT_ATTN_OK; ++k)
    for (int b = 0; b < 2; ++b)
      if (cudaEventCreateWithFlags(&ev[k][b], cudaEventDisableTiming) != cudaSuccess) rc = VGGT_ATTN_ERR_CUDA;
  const WorkspaceView w = workspace_view(shape, mode, workspace);
  const size_t row_bytes = static_cast<size_t>(shape->H) * 128;
  for (int i = 0; i < n_items && rc == VGGT_ATTN_OK; ++i) {
    const int b = i & 1;
    // H2D of item i into set b, after item i-2's kernels have read it.
    if (i >= 2 && cudaStreamWaitEvent(si, ev[1][b], 0) != cudaSuccess) { rc = VGGT_ATTN_ERR_CUDA; break; }
    if (cudaMemcpyAsync(P.qkv[b], h_qkv[i], P.qkv_bytes, cudaMemcpyHostToDevice, si) != cudaSuccess ||
        cudaEventRecord(ev[0][b], si) != cudaSuccess) { rc = VGGT_ATTN_ERR_CUDA; break; }
    // Kernels of item i, after its H2D and after item i-2's D2H has read out set b.
    if (cudaStreamWaitEvent(sc, ev[0][b], 0) != cudaSuccess ||
        (i >= 2 && cudaStreamWaitEvent(sc, ev[2][b], 0) != cudaSuccess)) { rc = VGGT_ATTN_ERR_CUDA; break; }
    if ((rc = launch_prologue(mode, shape, P.qkv[b], q_gamma, q_beta, k_gamma, k_beta, w, sc, i == 0))) break;
    if ((rc = launch_core(mode, shape, P.qkv[b], P.out[b], w, sc))) break;
    if (cudaEventRecord(ev[1][b], sc) != cudaSuccess) { rc = VGGT_ATTN_ERR_CUDA; break; }
    // D2H of item i (register mode: the special rows of every frame only).
    if (cudaStreamWaitEvent(so, ev[1][b], 0) != cudaSuccess) { rc = VGGT_ATTN_ERR_CUDA; break; }
    cudaError_t e;
    if (mode == VGGT_ATTN_REGISTER)
      e = cudaMemcpy2DAsync(h_out[i], shape->T * row_bytes, P.out[b], shape->T * row_bytes,
                            shape->n_special * row_bytes, shape->S, cudaMemcpyDeviceToHost, so);
    else
      e = cudaMemcpyAsync(h_out[i], P.out[b], P.out_bytes, cudaMemcpyDeviceToHost, so);
    if (e != cudaSuccess || cudaEventRecord(ev[2][b], so) != cudaSuccess) { rc = VGGT_ATTN_ERR_CUDA; break; }
  }
  for (int k = 0; k < 3; ++k)
    for (int b = 0; b < 2; ++b)
      if (ev[k][b]) cudaEventDestroy(ev[k][b]);   // released once the recorded work completes
  return rc;
}

// ---------------------------------------------------------------------------
// Query-sharded global attention, fused form: the core reads every rank's
// keys and values where the ranks' prologues wrote them (peer memory over
// NVLink for the other ranks), no gathered copy.
extern "C" size_t vggt_attn_shard_fused_workspace_size(const vggt_attn_shape* shape) {
  if (check_shard_shape(shape, 1) != VGGT_ATTN_OK) return 0;
  return static_cast<size_t>(reinterpret_cast<uintptr_t>(shard_layout(shape, 1, nullptr).k_all));
}

extern "C" int vggt_attn_global_shard_core_peers(const vggt_attn_shape* shape, int world, const void* const* k_ranks,
                                                 const void* const* v_ranks, void* out, void* workspace,
                                                 size_t workspace_bytes, void* cuda_stream) {
  int rc = check_shard_shape(shape, world);
  if (rc) return rc;
  if (world > vggt::kMaxRankMaps) return VGGT_ATTN_ERR_UNSUPPORTED_SHAPE;
  if ((rc = check_shard_ws(shape, world, workspace, workspace_bytes, true))) return rc;
  if (!out || !k_ranks || !v_ranks) return VGGT_ATTN_ERR_INVALID_ARG;
  for (int r = 0; r < world; ++r) {
    if (!k_ranks[r] || !v_ranks[r]) return VGGT_ATTN_ERR_INVALID_ARG;
    if (!aligned(k_ranks[r], 16) || !aligned(v_ranks[r], 16)) return VGGT_ATTN_ERR_MISALIGNED;
  }
  if (!aligned(out, 16)) return VGGT_ATTN_ERR_MISALIGNED;
  const size_t out_bytes = static_cast<size_t>(shape->S) * shape->T * shape->H * 128;
  if (overlaps(out, out_bytes, workspace, workspace_bytes)) return VGGT_ATTN_ERR_INVALID_ARG;
  if ((rc = check_device())) return rc;
  using C = vggt::CoreCfg<2, false, true, true>;
  const ShardLayout L = shard_layout(shape, world, workspace);
  const long long H = shape->H;
  CUtensorMap mq;
  {
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(L.L), static_cast<cuuint64_t>(H)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(L.L) * 128};
    const cuuint32_t box_q[3] = {64, vggt::core::BM, 1};
    if (!make_map(&mq, L.w.q, 3, dims, strides, box_q)) return VGGT_ATTN_ERR_CUDA;
  }
  vggt::RankMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  {
    // rank r's keys and values, [L][H][64]: (dim, head, token, 1); rows past L read as zeros
    const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(L.L), 1};
    const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128, static_cast<cuuint64_t>(L.L) * H * 128};
    const cuuint32_t box[4] = {64, 1, vggt::core::BN, 1};
    for (int r = 0; r < world; ++r)
      if (!make_map(&maps.k[r], k_ranks[r], 4, dims, strides, box) ||
          !make_map(&maps.v[r], v_ranks[r], 4, dims, strides, box))
        return VGGT_ATTN_ERR_CUDA;
  }
  const int spr = static_cast<int>((L.L + vggt::core::BN - 1) / vggt::core::BN);
  vggt::CoreParams p{};
  p.L = static_cast<int>(L.L);
  p.Lk = world * spr * vggt::core::BN;   // n_kv = world * spr steps
  p.H = shape->H;
  p.B = 1;
  p.out_T = shape->T;
  p.out_group = static_cast<int>(L.L);
  p.out = static_cast<uint16_t*>(out);
  p.out_elems = static_cast<long long>(shape->S) * shape->T * shape->H * 64;
  p.status = L.w.status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.rank_tokens = static_cast<int>(L.L);
  p.rank_steps = spr;
  if (cudaFuncSetAttribute(vggt::attn_core_ranks_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_ALLOC) != cudaSuccess)
    return VGGT_ATTN_ERR_CUDA;
  cudaFuncAttributes fa;   // the register split assumes the compiled count (see launch_core_cfg)
  if (cudaFuncGetAttributes(&fa, vggt::attn_core_ranks_kernel<C>) != cudaSuccess || fa.numRegs < C::REGS_AT_LAUNCH)
    return VGGT_ATTN_ERR_CUDA;
  const long long n_q = (L.L + 2 * vggt::core::BM - 1) / (2 * vggt::core::BM);
  const dim3 grid(static_cast<unsigned>(n_q), static_cast<unsigned>(H), 1);
  vggt::attn_core_ranks_kernel<C><<<grid, C::THREADS, C::SMEM_ALLOC, static_cast<cudaStream_t>(cuda_stream)>>>(
      mq, maps, p);
  return cudaGetLastError() == cudaSuccess ? VGGT_ATTN_OK : VGGT_ATTN_ERR_CUDA;
}
