"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
binding on seeded inputs and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import oracle as O
import workloads as W

MAX_ABS_TOL = 2e-2     # stated parity tolerance against the fp64 oracle
REL_FRO_TOL = 5e-3


def to_device(inputs):
    import torch
    dev = torch.device("cuda")
    qkv = torch.from_numpy(inputs["qkv"].view(np.int16)).to(dev).view(torch.bfloat16)
    params = {k: torch.from_numpy(np.ascontiguousarray(inputs[k])).to(dev)
              for k in ("q_gamma", "q_beta", "k_gamma", "k_beta")}
    return qkv, params


def run_gpu(mode, shape, inputs=None, dev_inputs=None, out=None, stream=None, check_status=True):
    """Run one mode through the binding; returns the bf16 ``out[S,T,H,64]`` tensor."""
    import torch
    import vit_attention_b200 as V
    qkv, prm = dev_inputs if dev_inputs is not None else to_device(inputs)
    if out is None:
        out = torch.empty((shape.S, shape.T, shape.H, 64), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(V.vggt_attn_workspace_size(shape, mode), dtype=torch.uint8, device="cuda")
    V.attend(mode, shape, qkv, prm["q_gamma"], prm["q_beta"], prm["k_gamma"], prm["k_beta"], out, ws, stream)
    if check_status:
        st = V.vggt_attn_read_status(ws, stream)
        assert st == 0, f"device status {st} ({V.error_string(st)})"
    torch.cuda.synchronize()
    return out


def rows(out, shape, flat_tokens):
    """fp64 numpy rows ``[n, H, 64]`` of the bf16 output for flat token indices."""
    import torch
    idx = torch.as_tensor(np.asarray(flat_tokens), device=out.device)
    return out.view(shape.S * shape.T, shape.H, 64).index_select(0, idx).float().cpu().numpy().astype(np.float64)


def errors(got, want):
    d = got - want
    return float(np.abs(d).max()), float(np.linalg.norm(d) / np.linalg.norm(want))


def assert_close(got, want, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs, rel = errors(got, want)
    assert max_abs <= MAX_ABS_TOL and rel <= REL_FRO_TOL, f"{what}: max_abs={max_abs:.3e} rel_fro={rel:.3e}"
    return max_abs, rel


def query_sample(mode, shape, count, seed):
    """Seeded query subset (flat token indices) valid for the mode."""
    if mode == "register":
        toks = O.register_tokens(shape)
        pick = W.query_subset(len(toks), count, seed)
        return toks[pick]
    return W.query_subset(shape.S * shape.T, count, seed)


def oracle_rows(mode, shape, inputs, queries, workers=None):
    """The oracle's rows for ``queries``, computed in query chunks on a thread
    pool (numpy releases the GIL in its array kernels; each chunk is an
    independent oracle call, and every query row is independent of the others,
    so the result equals one call on all queries)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    from threadpoolctl import threadpool_limits
    queries = np.asarray(queries, dtype=np.int64)
    workers = workers or os.cpu_count() or 1
    if len(queries) < 4096 or workers == 1:
        return O.attn_mode(mode, shape, inputs, queries)
    chunks = np.array_split(queries, 2 * workers)
    with threadpool_limits(1), ThreadPoolExecutor(workers) as ex:
        parts = list(ex.map(lambda c: O.attn_mode(mode, shape, inputs, c), chunks))
    return np.concatenate(parts, axis=0)


def check_mode(mode, shape, inputs, count=None, seed=0, out=None):
    """Run the GPU path, compare ``count`` sampled queries (all when None)."""
    out = run_gpu(mode, shape, inputs, out=out)
    q = query_sample(mode, shape, count if count is not None else 1 << 62, seed)
    want = oracle_rows(mode, shape, inputs, q)
    got = rows(out, shape, q)
    return assert_close(got, want, f"{mode} {shape}"), out
