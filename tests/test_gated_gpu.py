"""GPU parity of the gate formed in-kernel (gdn_chunk_fwd_gated, gdn_recurrent_step_gated).

The kernels receive the layer's raw projections a, b and the per-head
parameters A_log, dt_bias; the oracle forms g and beta with its own fp64 gate
function (oracle.gates: beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias),
walkthrough section 4) and runs the token recurrence.  Bars as in
test_parity_gpu.py: 1e-3 for fp32 q/k/v, 2e-2 for bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()


def _raw_gates(w, seed):
    """Per-head dt_bias ~ U(-1, 2) instead of the layer's initial 1, to exercise the bias."""
    gen = torch.Generator().manual_seed(seed)
    w["dt_bias"] = (torch.rand(w["nv"], generator=gen) * 3.0 - 1.0).contiguous()
    return w


def _oracle_gated(w):
    g, beta = oracle.gates(w["a"], w["b"], w["A_log"], w["dt_bias"])
    return oracle.recurrent(w["q"], w["k"], w["v"], g, beta, w["initial_state"], w["cu_seqlens"])


def _gpu_gated(w, chunk, kernel="auto"):
    from gated_deltanet_chunk_b200 import chunk_fwd_gated
    d = {k: (w[k].cuda() if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    out, sf = chunk_fwd_gated(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                              d["initial_state"], d["cu_seqlens"], chunk_size=chunk, kernel=kernel)
    torch.cuda.synchronize()
    return out, sf


@pytest.mark.parametrize("io,d,chunk,kernel", [("bf16", 128, 64, "tc"), ("bf16", 128, 64, "simt"),
                                               ("f32", 64, 64, "auto"), ("f32", 128, 128, "auto")])
def test_chunk_gated_against_oracle(io, d, chunk, kernel):
    lens = [1, 63, 64, 65, 200, 0, 777]
    w = _raw_gates(W.make_prefill(lengths=lens, nqk=2, nv=4, d=d, io=io, init_state=True, seed=41), 41)
    out, sf = _gpu_gated(w, chunk, kernel)
    ref_o, ref_s = _oracle_gated(w)
    U.check_prefill(out, sf, ref_o, ref_s, w["cu_seqlens"], U.TOL[io], "gated-" + kernel)


def test_chunk_gated_long_bf16_sampled_heads():
    """Full-size long prefill through the fused gate; the oracle checks 3 of the 32 v-heads."""
    w = W.make_workload("long_bf16_nv32", seed=42)
    out, sf = _gpu_gated(w, 64)
    heads = [0, 13, 31]
    G = w["nv"] // w["nqk"]
    sub = dict(q=w["q"][:, [h // G for h in heads]].contiguous(),
               k=w["k"][:, [h // G for h in heads]].contiguous(),
               v=w["v"][:, heads].contiguous(), a=w["a"][:, heads].contiguous(),
               b=w["b"][:, heads].contiguous(), A_log=w["A_log"][heads].contiguous(),
               dt_bias=w["dt_bias"][heads].contiguous(), initial_state=None,
               cu_seqlens=w["cu_seqlens"])
    ref_o, ref_s = _oracle_gated(sub)
    U.check_prefill(out[:, heads], sf[:, heads], ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"],
                    "gated-long")


def test_gated_equals_given_gates():
    """gdn_chunk_fwd_gated == gdn_chunk_fwd on the oracle's fp64 gates rounded to fp32."""
    from gated_deltanet_chunk_b200 import chunk_fwd
    w = _raw_gates(W.make_prefill(num_seqs=2, seq_len=500, nqk=2, nv=4, d=128, io="bf16",
                                  init_state=True, seed=43), 43)
    g64, b64 = oracle.gates(w["a"], w["b"], w["A_log"], w["dt_bias"])
    out1, sf1 = _gpu_gated(w, 64)
    dev = lambda x: torch.as_tensor(x, dtype=torch.float32).cuda().contiguous()
    out2, sf2 = chunk_fwd(w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), dev(g64), dev(b64),
                          w["initial_state"].cuda(), w["cu_seqlens"].cuda(), chunk_size=64)
    torch.cuda.synchronize()
    assert U.rel_inf(U.to_np(out1), U.to_np(out2)) < 1e-2
    assert U.rel_inf(U.to_np(sf1), U.to_np(sf2)) < 1e-3


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decode_gated_against_oracle(io):
    from gated_deltanet_chunk_b200 import recurrent_step_gated
    d = W.make_decode(num_seqs=64, steps=8, nqk=4, nv=8, io=io, seed=44)
    d["dt_bias"] = (torch.rand(8, generator=torch.Generator().manual_seed(44)) * 3.0 - 1.0)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    state = dev["initial_state"].clone()
    outs = []
    for t in range(d["steps"]):
        outs.append(recurrent_step_gated(dev["q"][t], dev["k"][t], dev["v"][t], dev["a"][t],
                                         dev["b"][t], dev["A_log"], dev["dt_bias"], state))
    torch.cuda.synchronize()
    steps, N = d["steps"], d["num_seqs"]
    pick = lambda t: t.transpose(0, 1).reshape(N * steps, *t.shape[2:]).cpu()
    g, beta = oracle.gates(pick(d["a"]), pick(d["b"]), d["A_log"].cpu(), d["dt_bias"].cpu())
    cu = torch.arange(N + 1, dtype=torch.int32) * steps
    ref_o, ref_s = oracle.recurrent(pick(d["q"]), pick(d["k"]), pick(d["v"]), g, beta,
                                    d["initial_state"].cpu(), cu)
    go = torch.stack(outs).transpose(0, 1).reshape(N * steps, 8, 128)
    U.check_prefill(go, state, ref_o, ref_s, cu, U.TOL[io], "decode-gated")
