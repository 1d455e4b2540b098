"""Helpers shared by the GPU parity tests: run the library and the oracle, compare.

Error metric (the reading used throughout): for each output tensor and for
each (sequence, v-head) slice of it, max|x - y| / max(max|y|, 1e-30) with y the
fp64 oracle.  Bars: 1e-3 when q, k, v are fp32; 2e-2 when they are bf16.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": 1e-3, "bf16": 2e-2}


def rel_inf(x, y) -> float:
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-30))


def to_np(t):
    return t.detach().float().cpu().double().numpy() if t is not None else None


def check_prefill(gpu_out, gpu_sf, ref_out, ref_sf, cu, tol, what=""):
    """Compare whole tensors and every (sequence, v-head) slice."""
    go, gs = to_np(gpu_out), to_np(gpu_sf)
    errs = {"out": rel_inf(go, ref_out)}
    if gs is not None:
        errs["final_state"] = rel_inf(gs, ref_sf)
    assert errs["out"] <= tol, (what, errs)
    if gs is not None:
        assert errs["final_state"] <= tol, (what, errs)
    cu = np.asarray(cu.cpu() if hasattr(cu, "cpu") else cu)
    worst = 0.0
    for n in range(len(cu) - 1):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        if sl.stop == sl.start:
            continue
        for h in range(ref_out.shape[1]):
            e = rel_inf(go[sl, h], ref_out[sl, h])
            worst = max(worst, e)
            assert e <= tol, (what, "out slice", n, h, e)
            if gs is not None:
                e2 = rel_inf(gs[n, h], ref_sf[n, h])
                worst = max(worst, e2)
                assert e2 <= tol, (what, "state slice", n, h, e2)
    errs["worst_slice"] = worst
    return errs


def run_gpu_prefill(w, chunk, kernel="auto", device="cuda"):
    from gated_deltanet_chunk_b200 import chunk_fwd
    d = {k: (w[k].to(device) if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    out, sf = chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"],
                        d["cu_seqlens"], chunk_size=chunk, kernel=kernel)
    torch.cuda.synchronize()
    return out, sf


def run_oracle_prefill(w):
    return oracle.recurrent(w["q"], w["k"], w["v"], w["g"], w["beta"], w["initial_state"],
                            w["cu_seqlens"])


def head_slice(w, heads):
    """Inputs of the chosen v-heads only (their qk-heads gathered): Nqk = Nv = len(heads)."""
    G = w["nv"] // w["nqk"]
    qk = [h // G for h in heads]
    s0 = w["initial_state"]
    return dict(q=w["q"][:, qk].contiguous(), k=w["k"][:, qk].contiguous(),
                v=w["v"][:, heads].contiguous(), g=w["g"][:, heads].contiguous(),
                beta=w["beta"][:, heads].contiguous(),
                initial_state=(s0[:, heads].contiguous() if s0 is not None else None),
                cu_seqlens=w["cu_seqlens"])
