"""The debug build (libvggt_attn_debug.so, compiled with -DVGGT_DEBUG): the same kernels with device-side
bounds checks on their direct global accesses, each of which records VGGT_ATTN_ERR_BOUNDS in the status word
and skips the access instead of faulting.  On valid inputs no check may fire and the results must be the
release build's: the test runs parity cases of every mode and a transformer block through the debug library
in a child process (VGGT_ATTN_LIBRARY=debug) and expects status 0 and the parity tolerance."""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys
    sys.path[:0] = [{root!r}, {tests!r}]
    import numpy as np, torch
    import vit_attention_b200 as V
    assert V.LIB_PATH.endswith("libvggt_attn_debug.so"), V.LIB_PATH
    import oracle as O, workloads as W
    from parity import check_mode
    def shp(S, H, ns, gh, gw): return W.Shape(S=S, T=ns + gh * gw, H=H, n_special=ns, grid_h=gh, grid_w=gw)
    for mode, s in [("frame", shp(3, 2, 17, 10, 30)), ("global", shp(4, 2, 3, 16, 16)),
                    ("register", shp(40, 2, 17, 4, 4)), ("frame", shp(300, 1, 2, 8, 16)), ("global", shp(2, 4, 5, 8, 8))]:
        (mx, rel), _ = check_mode(mode, s, W.make_random_inputs(s, 77 + s.T))
        print(mode, s.T, mx, rel)
    s = shp(3, 4, 5, 7, 9)
    w = W.make_transformer_block_weights(s.H, 5)
    x = W.make_tokens(s, 6)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).clone()
    dev = {{k: (torch.from_numpy(np.ascontiguousarray(v).view(np.int16)).cuda().view(torch.bfloat16)
               if v.dtype == np.uint16 else torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda())
           for k, v in w.items()}}
    ws = torch.empty(V.vggt_block_workspace_size(s, "global"), dtype=torch.uint8, device="cuda")
    V.vggt_block_forward("global", s, xd, dev, 1e-6, ws)
    assert V.vggt_attn_read_status(ws) == 0
    got = xd.double().cpu().numpy(); want = O.block_forward("global", s, x, w, 1e-6)
    assert np.linalg.norm(got - want) / np.linalg.norm(want) < 1e-2
    print("DEBUG BUILD OK")
""")


def test_debug_build_runs_every_mode_clean():
    lib = os.path.join(ROOT, "vit_attention_b200", "libvggt_attn_debug.so")
    if not os.path.exists(lib):
        import importlib.util
        spec = importlib.util.spec_from_file_location("_b", os.path.join(ROOT, "vit_attention_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build(debug=True)
    env = dict(os.environ, VGGT_ATTN_LIBRARY="debug")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"))
    res = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-4000:]
    assert "DEBUG BUILD OK" in res.stdout
