"""Python binding of libvggt_attn.so (argument marshalling only).

Every function here has the name of the C entry point it wraps (see
include/vggt_attn.h) and only converts arguments: tensors become device
pointers, the shape becomes the C struct, the stream defaults to torch's
current stream.  All computation runs in the library's CUDA kernels; there is
no fallback.  Importing this package fails loudly when the library has not
been built (``python -m vit_attention_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# VGGT_ATTN_LIBRARY=debug loads the debug build (device-side bounds checks, `build.py --debug`) instead.
LIB_PATH = os.path.join(_HERE, "libvggt_attn_debug.so" if os.environ.get("VGGT_ATTN_LIBRARY") == "debug"
                        else "libvggt_attn.so")

FRAME, GLOBAL, REGISTER = 0, 1, 2
MODES = {"frame": FRAME, "global": GLOBAL, "register": REGISTER}

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_SHAPE = -2
ERR_MISALIGNED = -3
ERR_WORKSPACE_TOO_SMALL = -4
ERR_CUDA = -5
ERR_TIMEOUT = -6
ERR_UNSUPPORTED_DEVICE = -7
ERR_SCRATCH_TOO_SMALL = -8
ERR_BOUNDS = -9
NOALLOC_SCRATCH_BYTES = 64 << 20


class vggt_attn_shape(ctypes.Structure):  # noqa: N801 - C name
    _fields_ = [("S", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("n_special", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("ln_eps", ctypes.c_float), ("rope_base", ctypes.c_float), ("softmax_scale", ctypes.c_float)]


BLOCK_WEIGHT_FIELDS = ("norm1_gamma", "norm1_beta", "w_qkv", "b_qkv", "q_gamma", "q_beta", "k_gamma", "k_beta",
                       "w_proj", "b_proj", "ls1", "norm2_gamma", "norm2_beta", "w_fc1", "b_fc1", "w_fc2", "b_fc2",
                       "ls2")


class vggt_block_weights(ctypes.Structure):  # noqa: N801 - C name
    _fields_ = [(f, ctypes.c_void_p) for f in BLOCK_WEIGHT_FIELDS]


class VggtAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {code} ({error_string(code)})")


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m vit_attention_b200.build` "
                      "(the CUDA library is required; there is no CPU path)")
_lib = ctypes.CDLL(LIB_PATH)

_vp, _sz, _int = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_shape_p = ctypes.POINTER(vggt_attn_shape)
_fp = ctypes.c_void_p  # float* passed as a raw device address
_MODE_SIG = [_shape_p, _vp, _fp, _fp, _fp, _fp, _vp, _vp, _sz, _vp]
_SIGNATURES = {
    "vggt_attn_workspace_size": (_sz, [_shape_p, _int]),
    "vggt_attn_frame": (_int, _MODE_SIG),
    "vggt_attn_global": (_int, _MODE_SIG),
    "vggt_attn_register": (_int, _MODE_SIG),
    "vggt_attn_prologue": (_int, [_int, _shape_p, _vp, _fp, _fp, _fp, _fp, _vp, _sz, _vp]),
    "vggt_attn_core": (_int, [_int, _shape_p, _vp, _vp, _vp, _sz, _vp]),
    "vggt_attn_read_status": (_int, [_vp, _vp, ctypes.POINTER(ctypes.c_int)]),
    "vggt_attn_selftest_timeout": (_int, [_vp, ctypes.c_uint, _vp]),
    "vggt_attn_error_string": (ctypes.c_char_p, [_int]),
    "vggt_attn_abi_version": (_int, []),
    "vggt_attn_noalloc": (_int, [_int, _shape_p, _vp, _fp, _fp, _fp, _fp, _vp, _vp]),
    "vggt_linear": (_int, [_int, _int, _int, _vp, _vp, _fp, _vp, _vp, _sz, _vp]),
    "vggt_attn_qkv_proj": (_int, [_int, _shape_p, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _vp, _vp, _sz, _vp]),
    "vggt_attn_block": (_int, [_int, _shape_p, _vp, _vp, _fp, _fp, _fp, _fp, _fp, _vp, _fp, _vp, _vp, _vp, _vp, _sz,
                               _vp]),
    "vggt_block_workspace_size": (_sz, [_shape_p, _int]),
    "vggt_block_forward": (_int, [_int, _shape_p, _vp, ctypes.POINTER(vggt_block_weights), ctypes.c_float, _vp, _sz,
                                  _vp]),
    "vggt_aggregator_workspace_size": (_sz, [_shape_p]),
    "vggt_aggregator_forward_cached": (_int, [_shape_p, _vp, ctypes.POINTER(vggt_block_weights),
                                              ctypes.POINTER(vggt_block_weights), _int, ctypes.POINTER(ctypes.c_int),
                                              _int, ctypes.POINTER(ctypes.c_int), _int, ctypes.POINTER(_vp),
                                              ctypes.c_float, _vp, _sz, _vp]),
    "vggt_aggregator_forward": (_int, [_shape_p, _vp, ctypes.POINTER(vggt_block_weights),
                                       ctypes.POINTER(vggt_block_weights), _int, ctypes.POINTER(ctypes.c_int), _int,
                                       ctypes.c_float, _vp, _sz, _vp]),
    "vggt_attn_host_pipeline_workspace_size": (_sz, [_shape_p, _int]),
    "vggt_attn_host_pipeline": (_int, [_int, _shape_p, _int, ctypes.POINTER(_vp), _fp, _fp, _fp, _fp,
                                       ctypes.POINTER(_vp), _vp, _sz, _vp, _vp, _vp]),
    "vggt_attn_shard_workspace_size": (_sz, [_shape_p, _int]),
    "vggt_attn_shard_buffers": (_int, [_shape_p, _int, _vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                       ctypes.POINTER(_vp), ctypes.POINTER(_vp)]),
    "vggt_attn_global_shard_prologue": (_int, [_shape_p, _int, _vp, _fp, _fp, _fp, _fp, _vp, _sz, _vp]),
    "vggt_attn_global_shard_core": (_int, [_shape_p, _int, _vp, _vp, _sz, _vp]),
    "vggt_attn_global_shard_core_local": (_int, [_shape_p, _int, _vp, _sz, _vp]),
    "vggt_attn_global_shard_core_remote": (_int, [_shape_p, _int, _int, _vp, _vp, _sz, _vp]),
    "vggt_attn_shard_fused_workspace_size": (_sz, [_shape_p]),
    "vggt_attn_global_shard_core_peers": (_int, [_shape_p, _int, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _vp,
                                                 _vp, _sz, _vp]),
    "vggt_camera_trunk_workspace_size": (_sz, [_shape_p]),
    "vggt_camera_trunk_forward": (_int, [_shape_p, _vp, _vp, ctypes.POINTER(vggt_block_weights), _int,
                                         ctypes.c_float, _vp, _sz, _vp]),
    "vggt_attn_sga_workspace_size": (_sz, [_shape_p, _int, _int]),
    "vggt_attn_global_sga": (_int, [_shape_p, _int, _int, _vp, _fp, _fp, _fp, _fp, _vp, _vp, _sz, _vp]),
    "vggt_attn_global_desc": (_int, [_shape_p, _int, _int, _vp, _fp, _fp, _fp, _fp, _vp, _vp, _sz, _vp]),
}
for _name, (_res, _args) in _SIGNATURES.items():
    _f = getattr(_lib, _name)
    _f.restype, _f.argtypes = _res, _args


def library():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib


def make_shape(shape) -> vggt_attn_shape:
    """C struct from any object with the struct's field names (or the struct itself)."""
    if isinstance(shape, vggt_attn_shape):
        return shape
    return vggt_attn_shape(shape.S, shape.T, shape.H, getattr(shape, "head_dim", 64), shape.n_special,
                           shape.grid_h, shape.grid_w, getattr(shape, "ln_eps", 1e-5),
                           getattr(shape, "rope_base", 100.0), getattr(shape, "softmax_scale", 0.0))


def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(ws, workspace_bytes):
    if workspace_bytes is not None:
        return workspace_bytes
    return ws.numel() * ws.element_size()


def _check(rc: int, where: str) -> None:
    if rc != OK:
        raise VggtAttnError(rc, where)


def error_string(code: int) -> str:
    return _lib.vggt_attn_error_string(code).decode()


def vggt_attn_abi_version() -> int:
    return _lib.vggt_attn_abi_version()


def vggt_attn_workspace_size(shape, mode) -> int:
    mode = MODES.get(mode, mode)
    return _lib.vggt_attn_workspace_size(ctypes.byref(make_shape(shape)), mode)


def _mode_call(fn, name, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes, stream):
    s = make_shape(shape)
    rc = fn(ctypes.byref(s), _ptr(qkv), _ptr(q_gamma), _ptr(q_beta), _ptr(k_gamma), _ptr(k_beta), _ptr(out),
            _ptr(workspace), _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, name)


def vggt_attn_frame(shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes=None, stream=None):
    _mode_call(_lib.vggt_attn_frame, "vggt_attn_frame", shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out,
               workspace, workspace_bytes, stream)


def vggt_attn_global(shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes=None, stream=None):
    _mode_call(_lib.vggt_attn_global, "vggt_attn_global", shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out,
               workspace, workspace_bytes, stream)


def vggt_attn_register(shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes=None,
                       stream=None):
    _mode_call(_lib.vggt_attn_register, "vggt_attn_register", shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out,
               workspace, workspace_bytes, stream)


def vggt_attn_prologue(mode, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace, workspace_bytes=None,
                       stream=None):
    mode = MODES.get(mode, mode)
    rc = _lib.vggt_attn_prologue(mode, ctypes.byref(make_shape(shape)), _ptr(qkv), _ptr(q_gamma), _ptr(q_beta),
                                 _ptr(k_gamma), _ptr(k_beta), _ptr(workspace), _nbytes(workspace, workspace_bytes),
                                 _stream(stream))
    _check(rc, "vggt_attn_prologue")


def vggt_attn_core(mode, shape, qkv, out, workspace, workspace_bytes=None, stream=None):
    mode = MODES.get(mode, mode)
    rc = _lib.vggt_attn_core(mode, ctypes.byref(make_shape(shape)), _ptr(qkv), _ptr(out), _ptr(workspace),
                             _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_core")


def vggt_attn_read_status(workspace, stream=None) -> int:
    st = ctypes.c_int(0)
    _check(_lib.vggt_attn_read_status(_ptr(workspace), _stream(stream), ctypes.byref(st)), "vggt_attn_read_status")
    return st.value


def vggt_attn_selftest_timeout(workspace, timeout_us: int, stream=None) -> None:
    _check(_lib.vggt_attn_selftest_timeout(_ptr(workspace), timeout_us, _stream(stream)),
           "vggt_attn_selftest_timeout")


def vggt_attn_noalloc(mode, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, stream=None):
    """Same computation as vggt_attn_{frame,global,register}, for callers that
    cannot give the library a workspace: the library uses its own fixed
    64 MiB device scratch instead (shared by all calls; serialise calls)."""
    mode = MODES.get(mode, mode)
    rc = _lib.vggt_attn_noalloc(mode, ctypes.byref(make_shape(shape)), _ptr(qkv), _ptr(q_gamma), _ptr(q_beta),
                                _ptr(k_gamma), _ptr(k_beta), _ptr(out), _stream(stream))
    _check(rc, "vggt_attn_noalloc")


_ENTRY = {"frame": vggt_attn_frame, "global": vggt_attn_global, "register": vggt_attn_register}


def attend(mode: str, shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, stream=None):
    """Dispatch by mode name to vggt_attn_{frame,global,register}."""
    _ENTRY[mode](shape, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, None, stream)


def vggt_linear(x, w, bias, y, workspace, workspace_bytes=None, stream=None):
    """y[M][N] = x[M][K] . w[N][K]^T + bias[N] (bf16 tensors, fp32 bias or None)."""
    M, K = x.shape[-2], x.shape[-1]
    N = w.shape[0]
    rc = _lib.vggt_linear(M, N, K, _ptr(x), _ptr(w), _ptr(bias), _ptr(y), _ptr(workspace),
                          _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_linear")


def vggt_attn_qkv_proj(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, qkv, workspace,
                       workspace_bytes=None, stream=None):
    mode = MODES.get(mode, mode)
    rc = _lib.vggt_attn_qkv_proj(mode, ctypes.byref(make_shape(shape)), _ptr(x), _ptr(w_qkv), _ptr(b_qkv),
                                 _ptr(q_gamma), _ptr(q_beta), _ptr(k_gamma), _ptr(k_beta), _ptr(qkv), _ptr(workspace),
                                 _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_qkv_proj")


def vggt_attn_block(mode, shape, x, w_qkv, b_qkv, q_gamma, q_beta, k_gamma, k_beta, w_out, b_out, qkv, attn, y,
                    workspace, workspace_bytes=None, stream=None):
    mode = MODES.get(mode, mode)
    rc = _lib.vggt_attn_block(mode, ctypes.byref(make_shape(shape)), _ptr(x), _ptr(w_qkv), _ptr(b_qkv),
                              _ptr(q_gamma), _ptr(q_beta), _ptr(k_gamma), _ptr(k_beta), _ptr(w_out), _ptr(b_out),
                              _ptr(qkv), _ptr(attn), _ptr(y), _ptr(workspace), _nbytes(workspace, workspace_bytes),
                              _stream(stream))
    _check(rc, "vggt_attn_block")


def vggt_attn_sga_workspace_size(shape, s_h: int, s_w: int) -> int:
    return _lib.vggt_attn_sga_workspace_size(ctypes.byref(make_shape(shape)), s_h, s_w)


def vggt_attn_global_sga(shape, s_h, s_w, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace, workspace_bytes=None,
                         stream=None):
    """Subsampled global attention: kept key grid s_h x s_w, diagonal, mean pair."""
    rc = _lib.vggt_attn_global_sga(ctypes.byref(make_shape(shape)), s_h, s_w, _ptr(qkv), _ptr(q_gamma), _ptr(q_beta),
                                   _ptr(k_gamma), _ptr(k_beta), _ptr(out), _ptr(workspace),
                                   _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_global_sga")


def make_block_weights(w) -> vggt_block_weights:
    """C struct of device addresses from a mapping with the struct's field names (tensors, ints or None)."""
    if isinstance(w, vggt_block_weights):
        return w
    return vggt_block_weights(*[_ptr(w.get(f)) for f in BLOCK_WEIGHT_FIELDS])


def vggt_block_workspace_size(shape, mode) -> int:
    mode = MODES.get(mode, mode)
    return _lib.vggt_block_workspace_size(ctypes.byref(make_shape(shape)), mode)


def vggt_block_forward(mode, shape, x, weights, norm_eps, workspace, workspace_bytes=None, stream=None):
    """One pre-norm transformer block applied in place to x [S][T][C] (bf16)."""
    mode = MODES.get(mode, mode)
    w = make_block_weights(weights)
    rc = _lib.vggt_block_forward(mode, ctypes.byref(make_shape(shape)), _ptr(x), ctypes.byref(w), norm_eps,
                                 _ptr(workspace), _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_block_forward")


def vggt_aggregator_workspace_size(shape) -> int:
    return _lib.vggt_aggregator_workspace_size(ctypes.byref(make_shape(shape)))


def vggt_aggregator_forward_cached(shape, x, frame_blocks, inter_blocks, register_layers, cache, norm_eps,
                                   workspace, workspace_bytes=None, stream=None):
    """vggt_aggregator_forward, also keeping the features of the layers in ``cache`` (a dict layer -> bf16
    device tensor [S*T, 2C]): frame-block output in the first C channels, inter-frame-block output in the rest."""
    n = len(frame_blocks)
    if len(inter_blocks) != n:
        raise ValueError("frame_blocks and inter_blocks must have one entry per layer")
    fb = (vggt_block_weights * max(n, 1))(*[make_block_weights(w) for w in frame_blocks])
    ib = (vggt_block_weights * max(n, 1))(*[make_block_weights(w) for w in inter_blocks])
    regs = (ctypes.c_int * max(len(register_layers), 1))(*register_layers)
    layers = sorted(cache)
    cl = (ctypes.c_int * max(len(layers), 1))(*layers)
    co = (_vp * max(len(layers), 1))(*[_ptr(cache[l]) for l in layers])
    rc = _lib.vggt_aggregator_forward_cached(ctypes.byref(make_shape(shape)), _ptr(x), fb, ib, n, regs,
                                             len(register_layers), cl, len(layers), co, norm_eps, _ptr(workspace),
                                             _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_aggregator_forward_cached")


def vggt_aggregator_forward(shape, x, frame_blocks, inter_blocks, register_layers, norm_eps, workspace,
                            workspace_bytes=None, stream=None):
    """Alternating frame / inter-frame blocks applied in place to x; inter-frame blocks of the layers in
    register_layers run in register mode, the others in global mode."""
    n = len(frame_blocks)
    if len(inter_blocks) != n:
        raise ValueError("frame_blocks and inter_blocks must have one entry per layer")
    fb = (vggt_block_weights * max(n, 1))(*[make_block_weights(w) for w in frame_blocks])
    ib = (vggt_block_weights * max(n, 1))(*[make_block_weights(w) for w in inter_blocks])
    regs = (ctypes.c_int * max(len(register_layers), 1))(*register_layers)
    rc = _lib.vggt_aggregator_forward(ctypes.byref(make_shape(shape)), _ptr(x), fb, ib, n, regs,
                                      len(register_layers), norm_eps, _ptr(workspace),
                                      _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_aggregator_forward")


def vggt_camera_trunk_workspace_size(shape) -> int:
    return _lib.vggt_camera_trunk_workspace_size(ctypes.byref(make_shape(shape)))


def vggt_camera_trunk_forward(shape, feats, tokens, blocks, norm_eps, workspace, workspace_bytes=None, stream=None):
    """Gather the special tokens of feats [S][T][C] into tokens [S*n_special][C], then apply the blocks
    (global attention among those tokens) to tokens in place."""
    n = len(blocks)
    arr = (vggt_block_weights * max(n, 1))(*[make_block_weights(w) for w in blocks])
    rc = _lib.vggt_camera_trunk_forward(ctypes.byref(make_shape(shape)), _ptr(feats), _ptr(tokens), arr, n,
                                        norm_eps, _ptr(workspace), _nbytes(workspace, workspace_bytes),
                                        _stream(stream))
    _check(rc, "vggt_camera_trunk_forward")


def vggt_attn_shard_workspace_size(shape, world: int) -> int:
    return _lib.vggt_attn_shard_workspace_size(ctypes.byref(make_shape(shape)), world)


def vggt_attn_shard_buffers(shape, world: int, workspace):
    """Views (bf16 tensors) of the send and gathered k/v buffers inside a uint8 workspace tensor:
    (k_send, v_send, k_all, v_all), shapes [S*T, H, 64] and [world*S*T, H, 64]."""
    import torch
    ptrs = [ctypes.c_void_p() for _ in range(4)]
    rc = _lib.vggt_attn_shard_buffers(ctypes.byref(make_shape(shape)), world, _ptr(workspace),
                                      *[ctypes.byref(p) for p in ptrs])
    _check(rc, "vggt_attn_shard_buffers")
    n = shape.S * shape.T
    views = []
    for p, rows in zip(ptrs, (n, n, world * n, world * n)):
        off = p.value - workspace.data_ptr()
        nbytes = rows * shape.H * 64 * 2
        if off + nbytes > workspace.numel():     # a fused-size workspace has no gathered buffers
            views.append(None)
            continue
        views.append(workspace[off:off + nbytes].view(torch.bfloat16).view(rows, shape.H, 64))
    return tuple(views)


def vggt_attn_shard_fused_workspace_size(shape) -> int:
    return _lib.vggt_attn_shard_fused_workspace_size(ctypes.byref(make_shape(shape)))


def vggt_attn_global_shard_core_peers(shape, world, k_ranks, v_ranks, out, workspace, workspace_bytes=None,
                                      stream=None):
    """Core of query-sharded global attention reading every rank's keys/values in place: k_ranks[r] /
    v_ranks[r] are device addresses (ints or tensors) of rank r's send buffers, valid in this process."""
    if len(k_ranks) != world or len(v_ranks) != world:
        raise ValueError("one key and one value buffer per rank")
    ks = (_vp * world)(*[_ptr(t) for t in k_ranks])
    vs = (_vp * world)(*[_ptr(t) for t in v_ranks])
    rc = _lib.vggt_attn_global_shard_core_peers(ctypes.byref(make_shape(shape)), world, ks, vs, _ptr(out),
                                                _ptr(workspace), _nbytes(workspace, workspace_bytes),
                                                _stream(stream))
    _check(rc, "vggt_attn_global_shard_core_peers")


def vggt_attn_global_shard_prologue(shape, world, qkv, q_gamma, q_beta, k_gamma, k_beta, workspace,
                                    workspace_bytes=None, stream=None):
    rc = _lib.vggt_attn_global_shard_prologue(ctypes.byref(make_shape(shape)), world, _ptr(qkv), _ptr(q_gamma),
                                              _ptr(q_beta), _ptr(k_gamma), _ptr(k_beta), _ptr(workspace),
                                              _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_global_shard_prologue")


def vggt_attn_global_shard_core(shape, world, out, workspace, workspace_bytes=None, stream=None):
    rc = _lib.vggt_attn_global_shard_core(ctypes.byref(make_shape(shape)), world, _ptr(out), _ptr(workspace),
                                          _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_global_shard_core")


def vggt_attn_global_shard_core_local(shape, world, workspace, workspace_bytes=None, stream=None):
    """Overlapped form, first half: the rank's queries over its own keys (send buffers) into the workspace's
    partial softmax state; runs while the all-gather fills the gathered buffers."""
    rc = _lib.vggt_attn_global_shard_core_local(ctypes.byref(make_shape(shape)), world, _ptr(workspace),
                                                _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_global_shard_core_local")


def vggt_attn_global_shard_core_remote(shape, world, rank, out, workspace, workspace_bytes=None, stream=None):
    """Overlapped form, second half (after the all-gather): the other ranks' keys, merged with the partial
    state of vggt_attn_global_shard_core_local, into out."""
    rc = _lib.vggt_attn_global_shard_core_remote(ctypes.byref(make_shape(shape)), world, rank, _ptr(out),
                                                 _ptr(workspace), _nbytes(workspace, workspace_bytes),
                                                 _stream(stream))
    _check(rc, "vggt_attn_global_shard_core_remote")


def vggt_attn_host_pipeline_workspace_size(shape, mode) -> int:
    mode = MODES.get(mode, mode)
    return _lib.vggt_attn_host_pipeline_workspace_size(ctypes.byref(make_shape(shape)), mode)


def vggt_attn_host_pipeline(mode, shape, h_qkv, q_gamma, q_beta, k_gamma, k_beta, h_out, workspace,
                            workspace_bytes=None, compute_stream=None, h2d_stream=None, d2h_stream=None):
    """Attend len(h_qkv) scenes whose qkv inputs and outputs are pinned host tensors; the copies of
    neighbouring scenes run on h2d_stream / d2h_stream during each scene's kernels on compute_stream.
    Returns after enqueueing: synchronise d2h_stream before reading h_out."""
    mode = MODES.get(mode, mode)
    n = len(h_qkv)
    if len(h_out) != n:
        raise ValueError("one output buffer per input")
    qs = (_vp * max(n, 1))(*[_ptr(t) for t in h_qkv])
    outs = (_vp * max(n, 1))(*[_ptr(t) for t in h_out])
    sc = _stream(compute_stream)
    rc = _lib.vggt_attn_host_pipeline(mode, ctypes.byref(make_shape(shape)), n, qs, _ptr(q_gamma), _ptr(q_beta),
                                      _ptr(k_gamma), _ptr(k_beta), outs, _ptr(workspace),
                                      _nbytes(workspace, workspace_bytes), sc,
                                      sc if h2d_stream is None else _stream(h2d_stream),
                                      sc if d2h_stream is None else _stream(d2h_stream))
    _check(rc, "vggt_attn_host_pipeline")


def vggt_attn_global_desc(shape, s_h, s_w, qkv, q_gamma, q_beta, k_gamma, k_beta, out, workspace,
                          workspace_bytes=None, stream=None):
    """Descriptor attention: every query over the per-frame descriptors (special tokens, s_h x s_w window means)."""
    rc = _lib.vggt_attn_global_desc(ctypes.byref(make_shape(shape)), s_h, s_w, _ptr(qkv), _ptr(q_gamma),
                                    _ptr(q_beta), _ptr(k_gamma), _ptr(k_beta), _ptr(out), _ptr(workspace),
                                    _nbytes(workspace, workspace_bytes), _stream(stream))
    _check(rc, "vggt_attn_global_desc")
