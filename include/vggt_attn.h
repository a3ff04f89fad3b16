/*
 * vggt_attn.h -- C ABI of libvggt_attn.so, the sm_100a (B200) attention core
 * of a VGGT-style alternating-attention block.
 *
 * What it computes (VGGT-Omega Aggregator explainer, sections 2 and 3):
 * for every token and head, q and k go through a LayerNorm over the 64 head
 * dimensions with a per-head affine ("use_qk_norm=True"), patch tokens are
 * rotated by a 2D rotary position embedding from their (row, col) in the
 * patch grid (re-applied at every layer; HTTM article, "04 method"), and then
 * exact softmax attention runs in one of three modes:
 *   frame    -- each frame's T tokens attend among themselves (section 3, step 1);
 *   global   -- all S*T tokens form one sequence (section 3, mode 1);
 *   register -- only the n_special camera + register tokens of every frame
 *               attend, over each other (section 3, mode 2).
 *
 * Conventions fixed by this library where the pages are silent:
 *   - LayerNorm: biased variance, epsilon = shape->ln_eps (> 0).
 *   - RoPE: dims [0,32) rotate by the patch row, [32,64) by the patch column;
 *     within each 32-dim half, pair (j, j+16), j in [0,16), rotates by angle
 *     pos * rope_base^(-2j/32), (a, b) -> (a cos - b sin, b cos + a sin).
 *     Token t >= n_special is patch p = t - n_special at row p / grid_w,
 *     col p % grid_w (0-based); tokens t < n_special are not rotated.  Every
 *     frame uses the same positions, in global mode too.
 *   - softmax scale: shape->softmax_scale, or 1/sqrt(64) when <= 0.
 *   - register mode writes only rows t < n_special of every frame of `out`;
 *     patch rows are left byte-for-byte untouched.
 *
 * Data layout (all device memory, caller-owned, row-major, no padding):
 *   qkv      bf16 [S][T][3][H][64]   (index 0 = q, 1 = k, 2 = v), 16-byte aligned
 *   q_gamma, q_beta, k_gamma, k_beta   fp32 [H][64], 16-byte aligned
 *   out      bf16 [S][T][H][64], 16-byte aligned, must not overlap qkv
 *   workspace  >= vggt_attn_workspace_size(shape, mode) bytes, 256-byte aligned;
 *              holds the normalised, rotated bf16 q and k (and, in register
 *              mode, the gathered v) plus a status word.  Its contents
 *              between calls are the library's; one workspace must not be used
 *              by two calls that may run concurrently.
 *
 * Numerics: q and k are normalised and rotated in fp32, then rounded to bf16
 * (q pre-multiplied by softmax_scale * log2(e)); scores accumulate in fp32 on
 * the tensor cores; the online softmax runs in fp32 with base-2 exponentials;
 * probabilities are rounded to bf16 for the P.V product (fp32 accumulate); the
 * output is rounded to bf16 (nearest even).
 *
 * Calls are asynchronous: they validate every argument on the host, enqueue
 * kernels on `cuda_stream` (a cudaStream_t; NULL = legacy default stream) and
 * return without synchronising.  They allocate nothing.  Argument errors are
 * reported before anything is enqueued, with no side effects.  A device-side
 * failure (a bounded wait inside a kernel that ran out) is recorded in the
 * workspace status word and read with vggt_attn_read_status().
 *
 * Thread safety: concurrent calls on different workspaces are safe.  The only
 * mutable global state is the shared scratch of vggt_attn_noalloc (below).
 */
#ifndef VGGT_ATTN_H
#define VGGT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define VGGT_ATTN_ABI_VERSION 4

/* Return codes (0 = success). */
enum {
  VGGT_ATTN_OK = 0,
  VGGT_ATTN_ERR_INVALID_ARG = -1,       /* NULL pointer, bad mode, overlapping buffers, non-finite scalar */
  VGGT_ATTN_ERR_UNSUPPORTED_SHAPE = -2, /* head_dim != 64, T != n_special + grid_h*grid_w, sizes out of range */
  VGGT_ATTN_ERR_MISALIGNED = -3,        /* a pointer lacks the alignment stated above */
  VGGT_ATTN_ERR_WORKSPACE_TOO_SMALL = -4,
  VGGT_ATTN_ERR_CUDA = -5,              /* a CUDA runtime/driver call or a launch failed */
  VGGT_ATTN_ERR_TIMEOUT = -6,           /* a bounded wait inside a kernel expired (vggt_attn_read_status) */
  VGGT_ATTN_ERR_UNSUPPORTED_DEVICE = -7, /* current device is not compute capability 10.0 (sm_100a) */
  VGGT_ATTN_ERR_SCRATCH_TOO_SMALL = -8,  /* vggt_attn_noalloc: the problem needs more than VGGT_ATTN_NOALLOC_SCRATCH_BYTES */
  VGGT_ATTN_ERR_BOUNDS = -9              /* debug build only (libvggt_attn_debug.so, -DVGGT_DEBUG): a device-side
                                            bounds check failed; the access was skipped, the status word records it */
};

/* Attention modes. */
enum { VGGT_ATTN_FRAME = 0, VGGT_ATTN_GLOBAL = 1, VGGT_ATTN_REGISTER = 2 };

typedef struct {
  int S;               /* frames, >= 1 */
  int T;               /* tokens per frame, >= 1 */
  int H;               /* heads, >= 1 */
  int head_dim;        /* must be 64 */
  int n_special;       /* camera + register tokens at the start of every frame, 0..T (>= 1 for register mode) */
  int grid_h, grid_w;  /* patch grid; T == n_special + grid_h * grid_w */
  float ln_eps;        /* QK-LayerNorm epsilon, > 0 */
  float rope_base;     /* RoPE base (100 for the VGGT-style aggregator), > 0 */
  float softmax_scale; /* <= 0 selects 1/sqrt(head_dim) */
} vggt_attn_shape;

/* Bytes of workspace a call in `mode` needs for `shape`; 0 if the shape or
 * mode is invalid. */
size_t vggt_attn_workspace_size(const vggt_attn_shape* shape, int mode);

/* Frame mode: each frame's tokens attend within the frame.  Writes all of `out`. */
int vggt_attn_frame(const vggt_attn_shape* shape, const void* qkv,
                    const float* q_gamma, const float* q_beta,
                    const float* k_gamma, const float* k_beta, void* out,
                    void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Global mode: all S*T tokens form one sequence.  Writes all of `out`. */
int vggt_attn_global(const vggt_attn_shape* shape, const void* qkv,
                     const float* q_gamma, const float* q_beta,
                     const float* k_gamma, const float* k_beta, void* out,
                     void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Register mode: the n_special tokens of every frame attend over the
 * S*n_special special tokens.  Writes only rows t < n_special of `out`. */
int vggt_attn_register(const vggt_attn_shape* shape, const void* qkv,
                       const float* q_gamma, const float* q_beta,
                       const float* k_gamma, const float* k_beta, void* out,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/* The two stages of the calls above, exposed so a caller can time or
 * schedule them separately.  vggt_attn_{frame,global,register} == prologue
 * followed by core on the same stream.
 *   prologue: QK-LayerNorm + RoPE of q and k (and, in register mode, the
 *             gather of the special tokens' v) into `workspace`; also clears
 *             the workspace status word.
 *   core:     attention over the packed workspace, writing `out`.
 * `qkv` is read by both stages (core reads v from it in frame/global mode). */
int vggt_attn_prologue(int mode, const vggt_attn_shape* shape, const void* qkv,
                       const float* q_gamma, const float* q_beta,
                       const float* k_gamma, const float* k_beta,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_core(int mode, const vggt_attn_shape* shape, const void* qkv, void* out,
                   void* workspace, size_t workspace_bytes, void* cuda_stream);

/* Synchronises `cuda_stream`, then reads and clears the status word of
 * `workspace`.  *status receives 0 or a negative VGGT_ATTN_ERR_* code
 * recorded by a kernel since the last prologue on this workspace.
 * Returns VGGT_ATTN_OK or VGGT_ATTN_ERR_CUDA / _INVALID_ARG. */
int vggt_attn_read_status(void* workspace, void* cuda_stream, int* status);

/* Fault-path self-test: launches one kernel whose bounded wait on an
 * mbarrier that nothing arrives at runs out after `timeout_us` microseconds
 * (1..1000000); it records VGGT_ATTN_ERR_TIMEOUT in the status word of
 * `workspace` (>= 256 bytes) and exits normally.  Used to test the error path
 * without faulting the GPU. */
int vggt_attn_selftest_timeout(void* workspace, unsigned timeout_us, void* cuda_stream);

/* Static, human-readable text for a return code. */
const char* vggt_attn_error_string(int code);

/* VGGT_ATTN_ABI_VERSION of the loaded library. */
int vggt_attn_abi_version(void);

/* ------------------------------------------------------------------------
 * Allocation-free variant (library addition; the pages have no counterpart).
 *
 * Some callers cannot hand the library a workspace: a plug-in interface that
 * passes only input and output buffers, code that must not call cudaMalloc or
 * cudaFree (cudaFree synchronises the whole device), or a process whose
 * device-memory budget is fixed at start-up.  vggt_attn_noalloc runs the same
 * prologue and attention kernels as vggt_attn_frame / _global / _register
 * (selected by `mode`), but its workspace is a fixed scratch array inside the
 * library: VGGT_ATTN_NOALLOC_SCRATCH_BYTES (64 MiB) of device memory that every
 * GPU which loads the library holds until the process exits.
 *
 *   - Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library
 *     routine.  The caller still owns and passes qkv, gamma/beta and out.
 *   - Problems whose workspace (vggt_attn_workspace_size) exceeds the scratch
 *     are rejected with VGGT_ATTN_ERR_SCRATCH_TOO_SMALL before anything runs.
 *     Global mode fits up to S*T*H ~ 262,000 token-heads (e.g. 15 frames of
 *     1031 tokens x 16 heads); register mode up to S*n_special*H ~ 174,000.
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it together
 *     with the id of the CUDA context it belongs to; make that first call
 *     before any stream capture on the device.  A device reset
 *     (cudaDeviceReset) unloads the library's module with the context: the
 *     cached address is then invalid, and the first call in the new context
 *     looks it up again (so, after a reset, that call too should come before
 *     any stream capture).
 *   - All calls share the one array, and it keeps the last call's contents
 *     (the prologue clears the status word each call; everything else is fully
 *     rewritten before it is read).  Calls that may overlap on the GPU -- on
 *     different streams, or from different threads without ordering -- race
 *     on it; serialise them.
 *   - A device-side timeout is recorded in the shared scratch; it is not
 *     readable through this entry point.
 * Arguments and errors are otherwise those of vggt_attn_frame. */
#define VGGT_ATTN_NOALLOC_SCRATCH_BYTES (64u << 20)
int vggt_attn_noalloc(int mode, const vggt_attn_shape* shape, const void* qkv,
                      const float* q_gamma, const float* q_beta,
                      const float* k_gamma, const float* k_beta, void* out,
                      void* cuda_stream);

/* ------------------------------------------------------------------------
 * Projections either side of the attention core (VGGT-Omega Aggregator
 * explainer, section 3: every attention block of the alternating-attention
 * layer projects its C = H*64 channels to q, k and v, and its attention output
 * back to C channels).  bf16 operands, fp32 accumulation on the tensor cores,
 * bf16 results rounded to nearest even.  Weights use the nn.Linear layout
 * [out_features][in_features]; biases are fp32 and may be NULL.
 *
 * vggt_linear: y[M][N] = x[M][K] . w[N][K]^T + bias[N].
 *   M >= 1, N a multiple of 256, K a multiple of 64 (K, N <= 65536).
 *   x, w, y, bias: 16-byte aligned; y must not overlap x or w.
 *   `workspace` (>= 256 bytes, 256-byte aligned) receives the status word of
 *   a device-side timeout (read with vggt_attn_read_status); it is not
 *   cleared by this call.
 *
 * vggt_attn_qkv_proj: the QKV projection of a frame- or global-mode block with
 * the prologue fused into it.  x is bf16 [S*T][C] (token features), w_qkv bf16
 * [3C][C], b_qkv fp32 [3C] or NULL.  The q and k columns of every head go
 * through the QK-LayerNorm, RoPE and softmax-scale step of vggt_attn_prologue
 * in fp32 straight from the accumulator (no bf16 rounding of the projection
 * before the LayerNorm) and land in `workspace`; the v columns are written to
 * the v slot of qkv [S][T][3][H][64] (its q and k slots are not written).
 * Afterwards vggt_attn_core(mode, shape, qkv, out, workspace, ...) computes
 * the attention exactly as after vggt_attn_prologue.  Requires H a multiple
 * of 4 (3C a multiple of 256); register mode is not supported
 * (VGGT_ATTN_ERR_INVALID_ARG).  Clears the workspace status word.
 *
 * vggt_attn_block: one attention block, y = (attention(x W_qkv^T + b_qkv))
 * W_out^T + b_out: vggt_linear of x into qkv (bf16 [S*T][3C]),
 * vggt_attn_prologue, vggt_attn_core into `attn` (bf16 [S*T][C]), then
 * vggt_linear with w_out [C][C], b_out [C] into y [S*T][C].  (The fused
 * vggt_attn_qkv_proj does less memory traffic but its LayerNorm/RoPE epilogue
 * sets its time; the unfused pair measured faster.)  `qkv` and `attn` are
 * caller-provided scratch; y must not overlap x, qkv, attn or the workspace.
 * Requires H a multiple of 4.  Register mode (workspace sized for register
 * mode; 3 n_special <= T): the block runs on the special tokens only -- their
 * rows of x are gathered, projected, attend over each other (register
 * attention), are projected back and scattered to their rows of y; patch
 * rows of y are not written, and attn holds the compact intermediates.
 *
 * All three are asynchronous on `cuda_stream`, validate every argument before
 * enqueueing anything and allocate nothing. */
int vggt_linear(int M, int N, int K, const void* x, const void* w, const float* bias, void* y,
                void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_qkv_proj(int mode, const vggt_attn_shape* shape, const void* x,
                       const void* w_qkv, const float* b_qkv,
                       const float* q_gamma, const float* q_beta,
                       const float* k_gamma, const float* k_beta, void* qkv,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_block(int mode, const vggt_attn_shape* shape, const void* x,
                    const void* w_qkv, const float* b_qkv,
                    const float* q_gamma, const float* q_beta,
                    const float* k_gamma, const float* k_beta,
                    const void* w_out, const float* b_out, void* qkv, void* attn, void* y,
                    void* workspace, size_t workspace_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------
 * Subsampled global attention (AVGGT article, section B, point 2, "SGA"): an
 * approximation of global mode that keeps every query but only a grid of
 * keys.  Kept keys K: every camera/register token (t < n_special) of every
 * frame and the patch tokens at (row, col) with row % s_h == 0 and
 * col % s_w == 0 (one per s_h x s_w window).  Discarded set D: the other
 * tokens.  Query i attends to K, to its own key when i is in D (the diagonal),
 * and to the mean over D of the normalised, rotated keys and of the values,
 * counted |D| - [i in D] times.  q/k normalisation, RoPE and the softmax scale
 * are those of global mode; s_h = s_w = 1 gives global attention.
 *
 * vggt_attn_sga_workspace_size: bytes of workspace for (shape, s_h, s_w), or 0
 * if invalid (s_h, s_w >= 1).
 * vggt_attn_global_sga: arguments as vggt_attn_global plus s_h, s_w (1..1024);
 * writes all of `out`; asynchronous, validates before enqueueing. */
size_t vggt_attn_sga_workspace_size(const vggt_attn_shape* shape, int s_h, int s_w);

/* Descriptor attention (FlashVGGT article, abstract): each frame is
 * compressed into descriptors -- its camera/register tokens, unchanged, and
 * one descriptor per s_h x s_w window of its patch grid (windows tile the grid
 * from (0, 0), the last ones may be smaller) whose key is the mean of the
 * window's normalised, rotated keys and whose value is the mean of its
 * values -- and every query (all S*T tokens, normalised and rotated as in
 * global mode) attends to the descriptors of all frames.  s_h = s_w = 1 is
 * global attention.  Arguments and workspace as vggt_attn_global_sga (the
 * workspace size is vggt_attn_sga_workspace_size(shape, s_h, s_w)); writes
 * all of `out`; asynchronous, validates before enqueueing. */
int vggt_attn_global_desc(const vggt_attn_shape* shape, int s_h, int s_w, const void* qkv,
                          const float* q_gamma, const float* q_beta,
                          const float* k_gamma, const float* k_beta, void* out,
                          void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_global_sga(const vggt_attn_shape* shape, int s_h, int s_w, const void* qkv,
                         const float* q_gamma, const float* q_beta,
                         const float* k_gamma, const float* k_beta, void* out,
                         void* workspace, size_t workspace_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------
 * Transformer blocks and the alternating-attention layer schedule
 * (VGGT-Omega Aggregator explainer, section 3: 24 layers, each a frame block
 * followed by an inter-frame block, the inter-frame block global except at the
 * register layers [2, 6, 9, 14, 20], where only the camera and register
 * tokens take part; QK normalisation on and LayerScale in every attention
 * block).  A block is the pre-norm transformer block of the backbone:
 *
 *   x <- x + ls1 * proj(attention(qkv(norm1(x))))
 *   x <- x + ls2 * fc2(GELU(fc1(norm2(x))))
 *
 * norm1/norm2: LayerNorm over the C = 64 H channels of a token (biased
 * variance, eps = norm_eps, fp32 arithmetic, bf16 result); qkv: [3C][C]
 * weight, outputs ordered q | k | v, each [H][64]; attention: the mode's
 * QK-LayerNorm, 2D RoPE and exact softmax attention of vggt_attn_frame /
 * vggt_attn_global; proj: [C][C]; fc1: [4C][C] (hidden width 4C); GELU the
 * exact erf form x * Phi(x); fc2: [C][4C]; ls1, ls2: per-channel LayerScale.
 * Intermediates (norm outputs, qkv, attention output, hidden activations)
 * are bf16; every GEMM accumulates in fp32 and its bias / GELU / LayerScale
 * and residual add are applied in fp32 before the one bf16 rounding.
 *
 * Weights: all device pointers, caller-owned, bf16 matrices in nn.Linear
 * layout [out][in], fp32 vectors; biases may be NULL (zero), every other
 * pointer is required and 16-byte aligned. */
typedef struct {
  const float* norm1_gamma; const float* norm1_beta;   /* [C] */
  const void* w_qkv; const float* b_qkv;               /* bf16 [3C][C], fp32 [3C] */
  const float* q_gamma; const float* q_beta;           /* QK-LayerNorm of q, [H][64] */
  const float* k_gamma; const float* k_beta;           /* QK-LayerNorm of k, [H][64] */
  const void* w_proj; const float* b_proj;             /* bf16 [C][C], fp32 [C] */
  const float* ls1;                                    /* [C] */
  const float* norm2_gamma; const float* norm2_beta;   /* [C] */
  const void* w_fc1; const float* b_fc1;               /* bf16 [4C][C], fp32 [4C] */
  const void* w_fc2; const float* b_fc2;               /* bf16 [C][4C], fp32 [C] */
  const float* ls2;                                    /* [C] */
} vggt_block_weights;

/* vggt_block_workspace_size: bytes of workspace vggt_block_forward needs for
 * (shape, mode), or 0 if the shape or mode is invalid.  It covers the
 * attention workspace and the bf16 intermediates (for register mode, of the
 * S n_special special tokens only).
 *
 * vggt_block_forward: one block applied in place to x, bf16 [S][T][C]
 * (C = 64 H, a multiple of 256, at most 2048).  Frame mode: attention within
 * each frame; global mode: over all S T tokens.  Register mode: the block
 * runs on the special tokens alone (their rows are gathered, go through the
 * whole block with global attention among them, unrotated, and are scattered
 * back); patch rows of x are left untouched.  Kernels: LayerNorm, QKV GEMM,
 * attention prologue and core, projection GEMM with the LayerScale residual
 * add in its epilogue, LayerNorm, fc1 GEMM with GELU in its epilogue, fc2 GEMM
 * with the LayerScale residual add; the first kernel clears the workspace
 * status word.  x must not overlap the workspace or any weight.
 *
 * vggt_aggregator_forward: n_layers layers applied in place to x; layer l runs
 * vggt_block_forward(FRAME, frame_blocks[l]) and then the inter-frame block
 * inter_blocks[l] in register mode if l is one of register_layers[0 ..
 * n_register) and in global mode otherwise.  frame_blocks and inter_blocks
 * are host arrays of n_layers weight sets; register_layers is a host array
 * (NULL when n_register is 0).  The workspace must hold
 * vggt_aggregator_workspace_size(shape) bytes, the larger of the frame and
 * global (and register) block needs.
 *
 * All are asynchronous on cuda_stream, validate every argument before
 * enqueueing anything and allocate nothing. */
size_t vggt_block_workspace_size(const vggt_attn_shape* shape, int mode);
int vggt_block_forward(int mode, const vggt_attn_shape* shape, void* x, const vggt_block_weights* w,
                       float norm_eps, void* workspace, size_t workspace_bytes, void* cuda_stream);
size_t vggt_aggregator_workspace_size(const vggt_attn_shape* shape);
int vggt_aggregator_forward(const vggt_attn_shape* shape, void* x, const vggt_block_weights* frame_blocks,
                            const vggt_block_weights* inter_blocks, int n_layers, const int* register_layers,
                            int n_register, float norm_eps, void* workspace, size_t workspace_bytes,
                            void* cuda_stream);
/* vggt_aggregator_forward_cached: the same schedule, and for each layer
 * cache_layers[i] (host array, n_cache entries) the layer's features are kept
 * in cache_out[i] (device, bf16 [S][T][2C]): channels [0, C) the output of its
 * frame block, channels [C, 2C) the output of its inter-frame block
 * (Aggregator explainer, section 4: the cached layers 4, 11, 17 and 23 feed the
 * heads with the frame and inter-frame outputs concatenated; the camera trunk
 * takes the last layer's).  cache_out buffers must not overlap x or the
 * workspace. */
int vggt_aggregator_forward_cached(const vggt_attn_shape* shape, void* x, const vggt_block_weights* frame_blocks,
                                   const vggt_block_weights* inter_blocks, int n_layers,
                                   const int* register_layers, int n_register, const int* cache_layers,
                                   int n_cache, void* const* cache_out, float norm_eps, void* workspace,
                                   size_t workspace_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------
 * Host-memory pipeline: n_items independent calls of one mode (frame, global
 * or register; one scene each, all of `shape`) whose qkv inputs and outputs
 * live in pinned host memory.  Item i's qkv (h_qkv[i], bf16
 * [S][T][3][H][64]) is copied to the device on h2d_stream, attended on
 * compute_stream (prologue + core, as vggt_attn_frame/global/register) and
 * its result copied back to h_out[i] (bf16 [S][T][H][64]) on d2h_stream;
 * two device staging sets in the workspace let the copies of items i+1 and
 * i-1 run during item i's kernels.  In register mode only the special-token
 * rows of h_out[i] are written (one strided copy).  q/k gamma/beta are
 * device pointers shared by all items.  The host buffers must be page-locked
 * (cudaHostAlloc / cudaHostRegister; VGGT_ATTN_ERR_INVALID_ARG otherwise)
 * and stay valid until d2h_stream has completed; the call returns after
 * enqueueing (the three streams may be the same stream, which serialises the
 * items).  The first kernel clears the workspace status word.  Workspace:
 * vggt_attn_host_pipeline_workspace_size(shape, mode) bytes. */
size_t vggt_attn_host_pipeline_workspace_size(const vggt_attn_shape* shape, int mode);
int vggt_attn_host_pipeline(int mode, const vggt_attn_shape* shape, int n_items, const void* const* h_qkv,
                            const float* q_gamma, const float* q_beta,
                            const float* k_gamma, const float* k_beta, void* const* h_out,
                            void* workspace, size_t workspace_bytes,
                            void* compute_stream, void* h2d_stream, void* d2h_stream);

/* ------------------------------------------------------------------------
 * Query-sharded global attention over `world` ranks (one GPU each).  Rank r
 * holds frames [r S, (r+1) S) of the scene, S = shape->S (the LOCAL frame
 * count; every rank the same): its queries attend to the keys of all world S
 * frames.  The exchange step is an all-gather of the normalised, rotated keys
 * and of the values; everything else is local.  Three calls per rank:
 *
 *   1. vggt_attn_global_shard_prologue: the global-mode prologue on the
 *      rank's qkv (bf16 [S][T][3][H][64]): q into the workspace's q plane,
 *      k (QK-LayerNorm + RoPE) and a copy of v token-major into the send
 *      buffers k_send, v_send (bf16 [S T][H][64] each).
 *   2. the caller all-gathers k_send -> k_all and v_send -> v_all (bf16
 *      [world S T][H][64], rank-major: rank r's block at token offset r S T),
 *      e.g. NCCL all-gather over NVLink; vggt_attn_shard_buffers gives the
 *      four buffers' addresses inside the workspace.
 *   3. vggt_attn_global_shard_core: the attention core of the rank's S T
 *      queries over all world S T keys into out (bf16 [S][T][H][64]).
 *
 * RoPE positions are per frame as in global mode, so the result equals rows
 * [r S T, (r+1) S T) of vggt_attn_global on the whole scene (bit for bit:
 * every query row sees the same keys in the same 64-key steps).  world = 1
 * is plain global attention with the copies in between.  The workspace
 * (vggt_attn_shard_workspace_size bytes) holds the status word, the q plane,
 * both send buffers, both gathered buffers and the partial softmax state of
 * the overlapped form (below); the first kernel of call 1
 * clears the status word.  Calls are asynchronous on cuda_stream, validate
 * every argument before enqueueing anything and allocate nothing;
 * vggt_attn_shard_buffers does no device work. */
size_t vggt_attn_shard_workspace_size(const vggt_attn_shape* shape, int world);
/* Fused form: no all-gather.  vggt_attn_global_shard_core_peers runs rank r's
 * queries over the keys and values of every rank read where each rank's
 * prologue left them: k_ranks[q] / v_ranks[q] (q = 0 .. world-1, world <= 8)
 * are device addresses, valid in this process, of rank q's k_send / v_send
 * (this rank's own, and the peers' mapped over NVLink, e.g. through CUDA IPC);
 * each rank's block of keys starts a new 64-key step, so results agree with
 * vggt_attn_global to rounding (bit for bit when world = 1).  The caller makes
 * sure every rank's prologue has completed before any rank's core starts and
 * that no prologue overwrites its buffers while a core may still read them.
 * Its workspace needs only the status word, q plane and send buffers:
 * vggt_attn_shard_fused_workspace_size(shape) bytes (the prologue accepts
 * that size too). */
size_t vggt_attn_shard_fused_workspace_size(const vggt_attn_shape* shape);
int vggt_attn_global_shard_core_peers(const vggt_attn_shape* shape, int world, const void* const* k_ranks,
                                      const void* const* v_ranks, void* out,
                                      void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_shard_buffers(const vggt_attn_shape* shape, int world, void* workspace, void** k_send,
                            void** v_send, void** k_all, void** v_all);
int vggt_attn_global_shard_prologue(const vggt_attn_shape* shape, int world, const void* qkv,
                                    const float* q_gamma, const float* q_beta,
                                    const float* k_gamma, const float* k_beta,
                                    void* workspace, size_t workspace_bytes, void* cuda_stream);
int vggt_attn_global_shard_core(const vggt_attn_shape* shape, int world, void* out,
                                void* workspace, size_t workspace_bytes, void* cuda_stream);
/* Overlapped form of step 3, so that the all-gather runs beside attention:
 *
 *   3a. vggt_attn_global_shard_core_local (right after the prologue, on the
 *       compute stream, while the all-gather of step 2 runs on another
 *       stream): the rank's queries over its OWN keys and values, read from
 *       k_send / v_send.  Writes no output: it leaves each query row's
 *       softmax state over those keys in the workspace (fp32: the 64
 *       unnormalised sums of 2^(s - m) v, their weight sum and the reference
 *       max m; the workspace of vggt_attn_shard_workspace_size holds it).
 *       Reads nothing the all-gather writes and writes nothing it reads.
 *   3b. vggt_attn_global_shard_core_remote (after the all-gather has
 *       completed): the queries over the other world - 1 ranks' blocks of
 *       k_all / v_all (rank `rank`'s own block is skipped), merging the state
 *       3a left (both scaled to the larger reference max and added) before
 *       the division by the row sum; writes out as step 3 does.
 *
 * The softmax over the union of the two key sets is the attention over all
 * keys (VGGT-Omega Aggregator explainer, section 3: global attention over
 * every frame's tokens); the result equals step 3's to rounding (different
 * 64-key step boundaries and the fp32 merge), not bit for bit.  3b needs
 * 2 <= world <= 9 (one tensor map per remote rank) and 0 <= rank < world,
 * else VGGT_ATTN_ERR_UNSUPPORTED_SHAPE / VGGT_ATTN_ERR_INVALID_ARG; with one
 * rank call step 3.  3b must follow 3a of the same workspace on the GPU
 * (same stream, or an event between them).  Cost: the two launches take
 * 4-7 % longer than step 3's one launch (100-frame scene, 2-5 ranks, B200),
 * so the overlap pays only where the all-gather takes longer than that. */
int vggt_attn_global_shard_core_local(const vggt_attn_shape* shape, int world, void* workspace,
                                      size_t workspace_bytes, void* cuda_stream);
int vggt_attn_global_shard_core_remote(const vggt_attn_shape* shape, int world, int rank, void* out,
                                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/* ------------------------------------------------------------------------
 * Camera-head trunk (VGGT-Omega Aggregator explainer, section 4: the camera
 * head takes the first 17 tokens of every frame -- camera and register
 * tokens -- from the last layer's features and mixes them across frames once
 * more with 4 self-attention blocks before reading out each frame's camera).
 *
 * vggt_camera_trunk_forward: gathers rows t < n_special of every frame of
 * feats (bf16 [S][T][Cf], Cf = 64 Hf, a multiple of 256, at most 2048; the
 * last layer's concatenated frame and global features, Cf = 2048 for the
 * 1024-channel backbone) into tokens (bf16 [S n_special][Cf], caller-owned),
 * then applies n_blocks transformer blocks (vggt_block_forward, global mode
 * over the S n_special tokens, which carry no RoPE position) to tokens in
 * place.  shape describes feats: shape->H = Hf, and its S, T, n_special, grid
 * and epsilons are those of the backbone.  blocks is a host array of n_blocks
 * weight sets of width Cf.  Workspace: vggt_camera_trunk_workspace_size(shape)
 * bytes.  Asynchronous on cuda_stream, validates every argument before
 * enqueueing anything, allocates nothing. */
size_t vggt_camera_trunk_workspace_size(const vggt_attn_shape* shape);
int vggt_camera_trunk_forward(const vggt_attn_shape* shape, const void* feats, void* tokens,
                              const vggt_block_weights* blocks, int n_blocks, float norm_eps,
                              void* workspace, size_t workspace_bytes, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* VGGT_ATTN_H */
