"""Plain fp64 CPU oracle for the alternating-attention core -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never calls it, and it shares no code with the CUDA path: the
two meet only in the seeded inputs of ``workloads``.

What it computes is the plain definition of the method -- the attention core
of the VGGT-Omega Aggregator's alternating-attention block (VGGT-Omega
Aggregator explainer, sections 2 and 3):

  1. bf16 inputs are widened exactly to fp64;
  2. per token and head, q and k each go through a LayerNorm over the 64 head
     dimensions with a per-head affine (section 3, "use_qk_norm=True");
  3. patch tokens are rotated by a 2D rotary position embedding from their
     (row, col) in the patch grid, re-applied at every layer (section 3;
     HTTM, "04 method", paragraph on the RoPE effect); camera and register
     tokens are not rotated;
  4. exact softmax attention (max-subtracted) in one of three key/query sets:
     frame (one frame), global (all S*T tokens), register (the n_special
     camera + register tokens of every frame; section 3, modes 1 and 2).

Readings where the pages are silent:
  * LayerNorm uses the biased variance and an epsilon passed by the caller
    (1e-5 by default).
  * RoPE: dims [0, 32) use the patch row, dims [32, 64) the patch column;
    inside each 32-dim half, frequency j in [0, 16) is base^(-2j/32) and pairs
    dims (j, j+16) ("rotate-half" pairing); a rotated pair (a, b) at angle
    theta becomes (a cos - b sin, b cos + a sin).  Positions are 0-based and
    identical in every frame, also in global mode.
  * softmax scale defaults to 1/sqrt(64).
  * register mode leaves the patch rows of the output untouched.

Every function here is pinned by ``tests/test_oracle.py`` against closed
forms, invariants and brute force, not against itself.
"""
from .attention import (  # noqa: F401
    bf16_to_f64,
    layer_norm,
    rope_frequencies,
    patch_row_col,
    rope_2d,
    normalized_tokens,
    softmax_attention,
    attn_frame,
    attn_global,
    attn_register,
    attn_mode,
    register_tokens,
    resolved_scale,
)
from .projection import attention_block, linear, projected_qkv  # noqa: F401
from .sga import attn_global_sga, sga_kept_tokens  # noqa: F401
from .descriptor import attn_global_desc, descriptor_windows  # noqa: F401
from .block import (  # noqa: F401
    CACHED_LAYERS,
    CAMERA_TRUNK_BLOCKS,
    N_LAYERS,
    camera_trunk_forward,
    REGISTER_LAYERS,
    aggregator_forward,
    block_forward,
    gelu,
    token_layer_norm,
)
