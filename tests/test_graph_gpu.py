"""CUDA-graph capture of the library's calls.

A serving loop replays a captured decode step (and fixed-shape prefills)
instead of launching every kernel from the host.  Every entry point launches
only on the stream it is given, allocates nothing and makes no synchronous
call, so it can be captured.  A replay must give bit-identical results to the
same calls made eagerly (the same kernels on the same inputs in the same
order), and it must read its input buffers when it runs, not when it was
captured.  The replays are also checked against the fp64 oracle (bf16 bar
2e-2, as max |x - y| / max |y|).
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


def test_decode_conv_then_step_graph_matches_eager_and_oracle():
    """Three decode steps, each the conv update (conv_state in place) then the recurrent step
    (state in place), captured once; replayed twice from reset states."""
    import gated_deltanet_chunk_b200 as gdn
    N, nqk, nv, D, steps = 16, 2, 4, 128, 3
    d = W.make_decode(num_seqs=N, steps=steps, nqk=nqk, nv=nv, d=D, io="bf16", seed=61)
    c = W.make_conv_inputs(N * steps, nqk, nv, D, D, 4, "bf16", seed=61, num_states=N)
    C = c["C"]
    x = c["x"].reshape(steps, N, C).cuda()
    g, beta = d["g"].cuda(), d["beta"].cuda()
    wt, b = c["weight"].cuda(), c["bias"].cuda()
    qb = torch.empty(N, nqk, D, dtype=torch.bfloat16, device="cuda")
    kb, vb = torch.empty_like(qb), torch.empty(N, nv, D, dtype=torch.bfloat16, device="cuda")

    def run(state, cst, outs):
        for t in range(steps):
            gdn.qkv_conv_update(x[t], wt, cst, nqk, nv, D, D, bias=b, out=(qb, kb, vb))
            gdn.recurrent_step(qb, kb, vb, g[t], beta[t], state, out=outs[t])

    s0, c0 = d["initial_state"].cuda(), c["state"].cuda()
    s_e, c_e = s0.clone(), c0.clone()
    o_e = [torch.empty(N, nv, D, dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    run(s_e, c_e, o_e)
    torch.cuda.synchronize()

    s_g, c_g = s0.clone(), c0.clone()
    o_g = [torch.empty_like(o) for o in o_e]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(s_g, c_g, o_g)
    torch.cuda.synchronize()
    assert torch.equal(s_g, s0) and torch.equal(c_g, c0)  # capturing ran nothing
    for _ in range(2):
        s_g.copy_(s0)
        c_g.copy_(c0)
        graph.replay()
        torch.cuda.synchronize()
        for t in range(steps):
            assert torch.equal(o_g[t], o_e[t]), t
        assert torch.equal(s_g, s_e) and torch.equal(c_g, c_e)

    # against the oracle: the conv over each sequence's 3 tokens, then the recurrence
    xs = c["x"].reshape(steps, N, C).transpose(0, 1).reshape(N * steps, C)
    cu = np.arange(N + 1, dtype=np.int32) * steps
    y, ref_cs = oracle.causal_conv1d(xs, c["weight"], c["bias"], cu, c["state"])
    qk = nqk * D
    T = N * steps
    q, k, v = y[:, :qk].reshape(T, nqk, D), y[:, qk:2 * qk].reshape(T, nqk, D), y[:, 2 * qk:].reshape(T, nv, D)
    per_seq = lambda a: a.transpose(0, 1).reshape(T, *a.shape[2:])
    o, sf = oracle.recurrent(q, k, v, per_seq(d["g"]), per_seq(d["beta"]), d["initial_state"], cu)
    go = torch.stack(o_g, 1).reshape(T, nv, D)
    assert U.rel_inf(U.to_np(go), o) <= U.TOL["bf16"]
    assert U.rel_inf(U.to_np(s_g), sf) <= U.TOL["bf16"]
    assert np.array_equal(U.to_np(c_g), ref_cs)


def test_prefill_graph_reads_inputs_at_replay():
    """A captured tensor-core prefill (packed varlen batch with initial states): the replay equals
    the eager call and the oracle, and after the inputs are overwritten in place a second replay
    computes the new inputs' result."""
    from gated_deltanet_chunk_b200 import chunk_fwd
    w = W.make_prefill(lengths=[300, 65, 190], nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=62)
    w2 = W.make_prefill(lengths=[300, 65, 190], nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=63)
    dv = {k: (w[k].cuda() if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    T = dv["q"].shape[0]
    n = dv["cu_seqlens"].numel() - 1

    def call(out, sf):
        chunk_fwd(dv["q"], dv["k"], dv["v"], dv["g"], dv["beta"], dv["initial_state"], dv["cu_seqlens"],
                  chunk_size=64, out=out, final_state=sf)

    o_e = torch.empty(T, 4, 128, dtype=torch.bfloat16, device="cuda")
    s_e = torch.empty(n, 4, 128, 128, dtype=torch.float32, device="cuda")
    call(o_e, s_e)
    torch.cuda.synchronize()
    o_g, s_g = torch.empty_like(o_e), torch.empty_like(s_e)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(o_g, s_g)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o_g, o_e) and torch.equal(s_g, s_e)
    ref_o, ref_s = U.run_oracle_prefill(w)
    U.check_prefill(o_g, s_g, ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"], "graph replay")

    for key in ("q", "k", "v", "g", "beta", "initial_state"):
        dv[key].copy_(w2[key].cuda())
    graph.replay()
    torch.cuda.synchronize()
    ref_o, ref_s = U.run_oracle_prefill(w2)
    U.check_prefill(o_g, s_g, ref_o, ref_s, w2["cu_seqlens"], U.TOL["bf16"], "graph replay, new inputs")
