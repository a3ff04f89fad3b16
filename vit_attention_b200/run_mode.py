"""Run one attention mode (or one transformer block) on seeded synthetic inputs of a workload's shape and
print the time per call -- a small driver for timing and for profiling a single kernel under ncu.

    python -m vit_attention_b200.run_mode --mode frame --workload 4 --frames 60 --calls 3
    python -m vit_attention_b200.run_mode --mode global --block --workload 2 --calls 2

Inputs are drawn on the device (normal qkv or token features; block weights with N(0, 1/fan_in)
matrices); the first call is a warm-up.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import sys


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--mode", choices=("frame", "global", "register"), default="frame")
    ap.add_argument("--workload", type=int, default=4, help="index into workloads.workload()")
    ap.add_argument("--frames", type=int, default=0, help="override the frame count S (0: keep)")
    ap.add_argument("--calls", type=int, default=3, help="timed calls after one warm-up call")
    ap.add_argument("--block", action="store_true", help="run a whole transformer block instead of attention")
    ap.add_argument("--sga", type=int, default=0, help="global mode as subsampled global attention, s x s grid")
    ap.add_argument("--desc", type=int, default=0, help="global mode as descriptor attention, s x s windows")
    args = ap.parse_args(argv)

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch

    import vit_attention_b200 as V
    import workloads as W

    torch.cuda.set_device(0)
    shape = W.workload(args.workload).shape
    if args.frames > 0:
        shape = dataclasses.replace(shape, S=args.frames)
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    H, C = shape.H, shape.H * 64
    if args.block:
        def mat(n_out, n_in):
            return (torch.randn((n_out, n_in), generator=g, device="cuda") / n_in ** 0.5).to(torch.bfloat16)

        def vec(n, centre):
            return centre + 0.1 * torch.randn(n, generator=g, device="cuda")

        w = dict(norm1_gamma=vec(C, 1.0), norm1_beta=vec(C, 0.0), w_qkv=mat(3 * C, C), b_qkv=vec(3 * C, 0.0),
                 q_gamma=vec(C, 1.0), q_beta=vec(C, 0.0), k_gamma=vec(C, 1.0), k_beta=vec(C, 0.0),
                 w_proj=mat(C, C), b_proj=vec(C, 0.0), ls1=vec(C, 1.0), norm2_gamma=vec(C, 1.0),
                 norm2_beta=vec(C, 0.0), w_fc1=mat(4 * C, C), b_fc1=vec(4 * C, 0.0), w_fc2=mat(C, 4 * C),
                 b_fc2=vec(C, 0.0), ls2=vec(C, 1.0))
        x = torch.randn((shape.S * shape.T, C), generator=g, device="cuda").to(torch.bfloat16)
        ws = torch.empty(V.vggt_block_workspace_size(shape, args.mode), dtype=torch.uint8, device="cuda")

        def call():
            V.vggt_block_forward(args.mode, shape, x, w, 1e-6, ws)
    else:
        qkv = torch.randn((shape.S, shape.T, 3, H, 64), generator=g, device="cuda").to(torch.bfloat16)
        prm = [(1.0 if k % 2 == 0 else 0.0) + 0.1 * torch.randn((H, 64), generator=g, device="cuda")
               for k in range(4)]
        out = torch.empty((shape.S, shape.T, H, 64), dtype=torch.bfloat16, device="cuda")
        if args.sga or args.desc:
            sz = args.sga or args.desc
            fn = V.vggt_attn_global_sga if args.sga else V.vggt_attn_global_desc
            ws = torch.empty(V.vggt_attn_sga_workspace_size(shape, sz, sz), dtype=torch.uint8, device="cuda")

            def call():
                fn(shape, sz, sz, qkv, *prm, out, ws)
        else:
            ws = torch.empty(V.vggt_attn_workspace_size(shape, args.mode), dtype=torch.uint8, device="cuda")

            def call():
                V.attend(args.mode, shape, qkv, *prm, out, ws)

    call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.calls):
        call()
    t1.record()
    t1.synchronize()
    status = V.vggt_attn_read_status(ws)
    print(json.dumps({"mode": args.mode, "block": args.block, "sga": args.sga, "desc": args.desc,
                      "S": shape.S, "T": shape.T, "H": H,
                      "ms_per_call": t0.elapsed_time(t1) / max(args.calls, 1), "status": status}))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
