"""GPU parity of the gated RMSNorm epilogue (NEXT-2): gdn_chunk_fwd_ex and
gdn_recurrent_step_ex with norm_z, and the standalone gdn_gated_rmsnorm.

The expected values are the fp64 oracle's gated RMSNorm (oracle.gated_rmsnorm:
RMSNormGated of the walkthrough, sections 1 and 6) applied to the oracle's own
token-loop outputs, on the same seeded inputs.  Bars as in test_parity_gpu.py:
1e-3 for fp32 q/k/v/z, 2e-2 for bf16.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()


def _gpu_normed(w, z, nw, chunk, kernel, eps=EPS):
    from gated_deltanet_chunk_b200 import chunk_fwd_ex
    d = {k: (w[k].cuda() if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    out, sf = chunk_fwd_ex(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"], d["cu_seqlens"],
                           chunk_size=chunk, kernel=kernel, norm_z=z.cuda(), norm_weight=nw.cuda(),
                           norm_eps=eps)
    torch.cuda.synchronize()
    return out, sf


@pytest.mark.parametrize("io,d,chunk,kernel", [("bf16", 128, 64, "tc"), ("bf16", 128, 64, "simt"),
                                               ("f32", 128, 64, "auto"), ("f32", 64, 128, "auto")])
def test_chunk_normed_against_oracle(io, d, chunk, kernel):
    lens = [1, 63, 64, 65, 200, 0, 777]
    w = W.make_prefill(lengths=lens, nqk=2, nv=4, d=d, io=io, init_state=True, seed=61)
    z, nw = W.make_norm_inputs(w["v"].shape, io, seed=61)
    out, sf = _gpu_normed(w, z, nw, chunk, kernel)
    ref_o, ref_s = U.run_oracle_prefill(w)
    ref_y = oracle.gated_rmsnorm(ref_o, z, nw, EPS)
    U.check_prefill(out, sf, ref_y, ref_s, w["cu_seqlens"], U.TOL[io], "normed-" + kernel)


def test_chunk_normed_equals_separate_epilogue():
    """gdn_chunk_fwd_ex with norm_z is gdn_chunk_fwd followed by gdn_gated_rmsnorm in
    place on the stored o: the two give the same bits."""
    from gated_deltanet_chunk_b200 import chunk_fwd, gated_rmsnorm
    w = W.make_prefill(num_seqs=2, seq_len=700, nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=62)
    z, nw = W.make_norm_inputs(w["v"].shape, "bf16", seed=62)
    y1, _ = _gpu_normed(w, z, nw, 64, "tc", eps=1e-3)
    d = {k: (w[k].cuda() if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    o, _ = chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["initial_state"], None, num_seqs=2,
                     chunk_size=64, kernel="tc")
    y2 = gated_rmsnorm(o, z.cuda(), nw.cuda(), 1e-3)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_chunk_normed_long_bf16_sampled_heads():
    """Full-size long prefill with the fused norm (tensor-core kernel); the oracle checks 3 heads."""
    w = W.make_workload("long_bf16_nv32", seed=42)
    z, nw = W.make_norm_inputs(w["v"].shape, "bf16", seed=42)
    out, sf = _gpu_normed(w, z, nw, 64, "auto")
    heads = [0, 13, 31]
    sub = U.head_slice(w, heads)
    ref_o, ref_s = U.run_oracle_prefill(sub)
    ref_y = oracle.gated_rmsnorm(ref_o, z[:, heads], nw, EPS)
    U.check_prefill(out[:, heads], sf[:, heads], ref_y, ref_s, w["cu_seqlens"], U.TOL["bf16"],
                    "normed-long")


def test_chunk_all_fusions_together():
    """Fused gate + slot pool + norm in one gdn_chunk_fwd_ex call (tensor-core kernel)."""
    from gated_deltanet_chunk_b200 import chunk_fwd_ex
    lens = [130, 1, 64, 257]
    w = W.make_prefill(lengths=lens, nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=63)
    z, nw = W.make_norm_inputs(w["v"].shape, "bf16", seed=63)
    P = 9
    ids = np.array([7, 2, 0, 5], dtype=np.int32)
    pool = torch.randn(P, 4, 128, 128, generator=torch.Generator().manual_seed(64)) * 0.1
    gpool = pool.cuda()
    d = {k: (w[k].cuda() if isinstance(w[k], torch.Tensor) else w[k]) for k in w}
    out, _ = chunk_fwd_ex(d["q"], d["k"], d["v"], d["a"], d["b"], gpool, d["cu_seqlens"], chunk_size=64,
                          kernel="tc", A_log=d["A_log"], dt_bias=d["dt_bias"],
                          slot_ids=torch.from_numpy(ids).cuda(), norm_z=z.cuda(), norm_weight=nw.cuda())
    torch.cuda.synchronize()
    g, beta = oracle.gates(w["a"], w["b"], w["A_log"], w["dt_bias"])
    s0 = pool[torch.as_tensor(ids.astype(np.int64))]
    ref_o, ref_s = oracle.recurrent(w["q"], w["k"], w["v"], g, beta, s0, w["cu_seqlens"])
    ref_y = oracle.gated_rmsnorm(ref_o, z, nw, EPS)
    U.check_prefill(out, gpool[torch.as_tensor(ids.astype(np.int64))], ref_y, ref_s, w["cu_seqlens"],
                    U.TOL["bf16"], "all-fusions")
    untouched = [s for s in range(P) if s not in ids]
    assert torch.equal(gpool[untouched].cpu(), pool[untouched])


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decode_normed_against_oracle(io):
    from gated_deltanet_chunk_b200 import recurrent_step_ex
    d = W.make_decode(num_seqs=64, steps=6, nqk=4, nv=8, io=io, seed=65)
    z, nw = W.make_norm_inputs(d["v"].shape, io, seed=65)  # [steps, N, Nv, Dv]
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    state = dev["initial_state"].clone()
    zc, nwc = z.cuda(), nw.cuda()
    outs = []
    for t in range(d["steps"]):
        outs.append(recurrent_step_ex(dev["q"][t], dev["k"][t], dev["v"][t], dev["g"][t], dev["beta"][t],
                                      state, norm_z=zc[t], norm_weight=nwc, norm_eps=EPS))
    torch.cuda.synchronize()
    steps, N = d["steps"], d["num_seqs"]
    pick = lambda x: x.transpose(0, 1).reshape(N * steps, *x.shape[2:]).cpu()
    cu = torch.arange(N + 1, dtype=torch.int32) * steps
    ref_o, ref_s = oracle.recurrent(pick(d["q"]), pick(d["k"]), pick(d["v"]), pick(d["g"]),
                                    pick(d["beta"]), d["initial_state"].cpu(), cu)
    ref_y = oracle.gated_rmsnorm(ref_o, pick(z), nw, EPS)
    go = torch.stack(outs).transpose(0, 1).reshape(N * steps, 8, 128)
    U.check_prefill(go, state, ref_y, ref_s, cu, U.TOL[io], "decode-normed")


@pytest.mark.parametrize("io,dim,rows", [("bf16", 128, 1), ("bf16", 128, 1000), ("bf16", 64, 777),
                                         ("f32", 128, 333), ("f32", 64, 4099), ("bf16", 128, 0)])
def test_standalone_gated_rmsnorm(io, dim, rows):
    from gated_deltanet_chunk_b200 import gated_rmsnorm
    dtype = torch.float32 if io == "f32" else torch.bfloat16
    gen = torch.Generator().manual_seed(66 + rows)
    o = (torch.randn(rows, dim, generator=gen) * torch.rand(rows, 1, generator=gen) * 4).to(dtype)
    z, nw = W.make_norm_inputs((rows, dim), io, seed=66 + rows)
    y = gated_rmsnorm(o.cuda(), z.cuda(), nw.cuda(), 1e-5)
    oc = o.cuda()
    y_in_place = gated_rmsnorm(oc, z.cuda(), nw.cuda(), 1e-5, out=oc)
    torch.cuda.synchronize()
    if rows == 0:
        return
    ref = oracle.gated_rmsnorm(o, z, nw, 1e-5)
    # per row: the bf16 / fp32 rounding of y relative to the row's largest value
    tol = 8e-3 if io == "bf16" else 1e-5
    err = np.max(np.abs(U.to_np(y) - ref), axis=1) / np.maximum(np.max(np.abs(ref), axis=1), 1e-30)
    assert float(err.max()) < tol
    assert torch.equal(y, y_in_place)
