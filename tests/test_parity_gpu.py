"""GPU parity: libgdn.so (through the C ABI) against the fp64 oracle.

All inputs are seeded and synthetic (workloads/).  Bars: max relative error
<= 1e-3 for fp32 q/k/v, <= 2e-2 for bf16, on `out` and `final_state`, per
tensor and per (sequence, v-head) slice.
"""
import numpy as np
import pytest
import torch

import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()


def _prefill_case(w, chunk, kernel="auto", what=""):
    out, sf = U.run_gpu_prefill(w, chunk, kernel)
    ref_o, ref_s = U.run_oracle_prefill(w)
    return U.check_prefill(out, sf, ref_o, ref_s, w["cu_seqlens"], U.TOL[w["io"]], what)


# ---------------------------------------------------------------- configurations
def test_tiny_f32_d64():
    w = W.make_workload("tiny_f32_d64", seed=0)
    _prefill_case(w, 64, what="tiny")


def test_batch_f32_d128_gqa_initial_state():
    w = W.make_workload("batch_f32_d128", seed=1)
    _prefill_case(w, 128, what="batch_f32")


def test_long_bf16_nv32_full_size():
    w = W.make_workload("long_bf16_nv32", seed=2)
    _prefill_case(w, 64, what="long_bf16")


def test_varlen_bf16_nv32_sampled_heads():
    """Full varlen batch on the GPU; the oracle recomputes 4 of the 32 v-heads."""
    w = W.make_workload("varlen_bf16_nv32", seed=3)
    out, sf = U.run_gpu_prefill(w, 64)
    heads = [0, 7, 18, 31]
    sub = U.head_slice(w, heads)
    ref_o, ref_s = U.run_oracle_prefill(sub)
    U.check_prefill(out[:, heads], sf[:, heads], ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"], "varlen")


# ---------------------------------------------------------------- edge cases
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("d,chunk,nqk,nv", [(64, 64, 1, 1), (64, 128, 2, 4), (128, 64, 1, 4),
                                             (128, 128, 4, 4)])
def test_edge_lengths(io, d, chunk, nqk, nv):
    lens = [1, 63, 64, 65, 127, 128, 129, 0, 2, 200]
    w = W.make_prefill(lengths=lens, nqk=nqk, nv=nv, d=d, io=io, init_state=True, seed=11)
    _prefill_case(w, chunk, what="edge")


@pytest.mark.parametrize("gate", ["zero", "mild", "beta1", "zero_beta1"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_stress_gates_long_memory(gate, io):
    """Slow or no decay, so the inter-chunk state hand-off matters (T = 4096)."""
    kw = dict(num_seqs=1, seq_len=4096, nqk=1, nv=2, d=128, io=io, init_state=True, seed=21)
    if gate == "mild":
        w = W.make_prefill(**kw, A_hi=1e-3)
    else:
        w = W.make_prefill(**kw, gate=gate)
    _prefill_case(w, 64, what="stress-" + gate)


def test_dk_ne_dv():
    w = W.make_prefill(num_seqs=2, seq_len=300, nqk=1, nv=2, d=128, dv=64, io="f32", init_state=True, seed=5)
    _prefill_case(w, 64, what="dk!=dv")
    w = W.make_prefill(num_seqs=2, seq_len=300, nqk=1, nv=2, d=64, dv=128, io="bf16", init_state=True, seed=6)
    _prefill_case(w, 128, what="dk!=dv")


# ---------------------------------------------------------------- state carry, aliasing
def test_split_and_carry_matches_unsplit():
    from gated_deltanet_chunk_b200 import chunk_fwd
    w = W.make_prefill(num_seqs=1, seq_len=1000, nqk=2, nv=4, d=128, io="bf16", init_state=True,
                       seed=7, device="cuda")
    full_o, full_s = chunk_fwd(w["q"], w["k"], w["v"], w["g"], w["beta"], w["initial_state"], chunk_size=64)
    for t in (64, 333):
        o1, s1 = chunk_fwd(w["q"][:t], w["k"][:t], w["v"][:t], w["g"][:t], w["beta"][:t],
                           w["initial_state"], chunk_size=64)
        o2, s2 = chunk_fwd(w["q"][t:].contiguous(), w["k"][t:].contiguous(), w["v"][t:].contiguous(),
                           w["g"][t:].contiguous(), w["beta"][t:].contiguous(), s1, chunk_size=64)
        torch.cuda.synchronize()
        assert U.rel_inf(U.to_np(torch.cat([o1, o2])), U.to_np(full_o)) < 2e-2
        assert U.rel_inf(U.to_np(s2), U.to_np(full_s)) < 2e-2


def test_in_place_state_and_no_final_state():
    from gated_deltanet_chunk_b200 import chunk_fwd
    w = W.make_prefill(num_seqs=3, seq_len=100, nqk=1, nv=2, d=64, io="f32", init_state=True,
                       seed=8, device="cuda")
    ref_o, ref_s = chunk_fwd(w["q"], w["k"], w["v"], w["g"], w["beta"], w["initial_state"],
                             chunk_size=64, num_seqs=3)
    st = w["initial_state"].clone()
    o, s = chunk_fwd(w["q"], w["k"], w["v"], w["g"], w["beta"], st, chunk_size=64, num_seqs=3,
                     final_state=st)
    o2, s2 = chunk_fwd(w["q"], w["k"], w["v"], w["g"], w["beta"], w["initial_state"], chunk_size=64,
                       num_seqs=3, output_final_state=False)
    torch.cuda.synchronize()
    assert s2 is None
    assert torch.equal(st, ref_s) and torch.equal(o, ref_o) and torch.equal(o2, ref_o)


def test_deterministic():
    w = W.make_prefill(num_seqs=2, seq_len=777, nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=9)
    o1, s1 = U.run_gpu_prefill(w, 64)
    o2, s2 = U.run_gpu_prefill(w, 64)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_chunk_size_invariance_on_gpu():
    w = W.make_prefill(num_seqs=1, seq_len=1000, nqk=1, nv=2, d=128, io="f32", init_state=True, seed=10,
                       A_hi=0.05)
    o64, s64 = U.run_gpu_prefill(w, 64)
    o128, s128 = U.run_gpu_prefill(w, 128)
    assert U.rel_inf(U.to_np(o64), U.to_np(o128)) < 1e-4
    assert U.rel_inf(U.to_np(s64), U.to_np(s128)) < 1e-4


# ---------------------------------------------------------------- decode
def _decode_oracle(d, seqs):
    """Oracle over `steps` tokens for the chosen sequences, as packed sequences."""
    steps = d["steps"]
    pick = lambda t: t[:, seqs].transpose(0, 1).reshape(len(seqs) * steps, *t.shape[2:]).cpu()
    cu = torch.arange(len(seqs) + 1, dtype=torch.int32) * steps
    return U.oracle.recurrent(pick(d["q"]), pick(d["k"]), pick(d["v"]), pick(d["g"]), pick(d["beta"]),
                              d["initial_state"][seqs].cpu(), cu)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decode_steps_all_sequences(io):
    from gated_deltanet_chunk_b200 import recurrent_step
    d = W.make_decode(num_seqs=256, steps=12, io=io, seed=4)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    state = dev["initial_state"].clone()
    outs = []
    for t in range(d["steps"]):
        outs.append(recurrent_step(dev["q"][t], dev["k"][t], dev["v"][t], dev["g"][t], dev["beta"][t], state))
    torch.cuda.synchronize()
    seqs = list(range(256))
    ref_o, ref_s = _decode_oracle(d, seqs)
    go = torch.stack(outs).transpose(0, 1).reshape(256 * d["steps"], 32, 128)
    cu = torch.arange(257, dtype=torch.int32) * d["steps"]
    U.check_prefill(go, state, ref_o, ref_s, cu, U.TOL[io], "decode")


def test_decode_1024_steps_sampled_sequences():
    from gated_deltanet_chunk_b200 import recurrent_step
    d = W.make_decode(num_seqs=256, steps=1024, io="bf16", seed=4, device="cuda")
    state = d["initial_state"].clone()
    seqs = [0, 1, 77, 255]
    outs = []
    for t in range(d["steps"]):
        o = recurrent_step(d["q"][t], d["k"][t], d["v"][t], d["g"][t], d["beta"][t], state)
        outs.append(o[seqs].clone())
    torch.cuda.synchronize()
    ref_o, ref_s = _decode_oracle(d, seqs)
    go = torch.stack(outs).transpose(0, 1).reshape(len(seqs) * 1024, 32, 128)
    cu = torch.arange(len(seqs) + 1, dtype=torch.int32) * 1024
    U.check_prefill(go, state[seqs], ref_o, ref_s, cu, U.TOL["bf16"], "decode1024")


def test_decode_equals_chunk_with_t1():
    """gdn_recurrent_step == gdn_chunk_fwd over N sequences of one token."""
    from gated_deltanet_chunk_b200 import chunk_fwd, recurrent_step
    d = W.make_decode(num_seqs=64, steps=1, nqk=4, nv=8, io="f32", seed=12, device="cuda")
    st = d["initial_state"].clone()
    o_step = recurrent_step(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], st)
    o_chk, s_chk = chunk_fwd(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0],
                             d["initial_state"], chunk_size=64, num_seqs=64)
    torch.cuda.synchronize()
    assert U.rel_inf(U.to_np(o_step), U.to_np(o_chk)) < 1e-5
    assert U.rel_inf(U.to_np(st), U.to_np(s_chk)) < 1e-5


# ---------------------------------------------------------------- tensor-core kernel
@pytest.mark.parametrize("lens,nqk,nv,init", [([64], 1, 1, False), ([1], 1, 1, True), ([65, 63], 1, 2, True),
                                              ([700, 130, 1], 2, 4, True), ([4096], 4, 8, True)])
def test_tc_kernel_against_oracle(lens, nqk, nv, init):
    w = W.make_prefill(lengths=lens, nqk=nqk, nv=nv, d=128, io="bf16", init_state=init, seed=31)
    _prefill_case(w, 64, kernel="tc", what="tc")


def test_tc_kernel_matches_simt_kernel():
    w = W.make_prefill(num_seqs=3, seq_len=1000, nqk=2, nv=4, d=128, io="bf16", init_state=True, seed=32,
                       A_hi=0.5)
    o_tc, s_tc = U.run_gpu_prefill(w, 64, kernel="tc")
    o_si, s_si = U.run_gpu_prefill(w, 64, kernel="simt")
    assert U.rel_inf(U.to_np(o_tc), U.to_np(o_si)) < 2e-2
    assert U.rel_inf(U.to_np(s_tc), U.to_np(s_si)) < 2e-2


def test_tc_device_status_clean():
    import gated_deltanet_chunk_b200 as g
    w = W.make_prefill(num_seqs=1, seq_len=200, nqk=1, nv=2, d=128, io="bf16", seed=33)
    U.run_gpu_prefill(w, 64, kernel="tc")
    assert g.device_status() == 0


# ---------------------------------------------------------------- maximum sequence count
@pytest.mark.parametrize("io,d,kernel", [("bf16", 128, "tc"), ("f32", 64, "auto")])
def test_max_num_seqs_prefill(io, d, kernel):
    """65535 sequences (the ABI's limit: one grid dimension per sequence) of 0-3 tokens,
    with initial states; every sequence checked against the oracle."""
    lens = torch.randint(0, 4, (65535,), generator=torch.Generator().manual_seed(91))
    w = W.make_prefill(lengths=lens, nqk=1, nv=1, d=d, io=io, init_state=True, seed=91)
    _prefill_case(w, 64, kernel, "max-seqs-" + kernel)


def test_max_num_seqs_decode():
    """One decode step for 65535 sequences (grid y = sequences)."""
    from gated_deltanet_chunk_b200 import recurrent_step
    d = W.make_decode(num_seqs=65535, steps=1, nqk=1, nv=1, d=64, io="bf16", seed=92)
    state = d["initial_state"].cuda()
    out = recurrent_step(d["q"][0].cuda(), d["k"][0].cuda(), d["v"][0].cuda(), d["g"][0].cuda(),
                         d["beta"][0].cuda(), state)
    torch.cuda.synchronize()
    import oracle
    cu = torch.arange(65536, dtype=torch.int32)
    ref_o, ref_s = oracle.recurrent(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0],
                                    d["initial_state"], cu)
    U.check_prefill(out, state, ref_o, ref_s, cu, U.TOL["bf16"], "max-seqs-decode")


@pytest.mark.parametrize("io,d,kernel", [("bf16", 128, "auto"), ("bf16", 128, "tc"), ("bf16", 128, "simt"),
                                         ("f32", 64, "auto")])
def test_empty_batch_copies_states(io, d, kernel):
    """total_tokens = 0 (three empty sequences): final_state = initial_state, bit for bit, for every
    kernel setting (the tensor-core setting included)."""
    from gated_deltanet_chunk_b200 import chunk_fwd
    dtype = torch.bfloat16 if io == "bf16" else torch.float32
    e = lambda *shape: torch.empty(*shape, dtype=dtype, device="cuda")
    s0 = torch.randn(3, 2, d, d, generator=torch.Generator().manual_seed(96)).cuda()
    g0 = torch.empty(0, 2, device="cuda")
    out, sf = chunk_fwd(e(0, 1, d), e(0, 1, d), e(0, 2, d), g0, g0.clone(), s0,
                        torch.zeros(4, dtype=torch.int32, device="cuda"), chunk_size=64, kernel=kernel)
    torch.cuda.synchronize()
    assert out.numel() == 0 and torch.equal(sf, s0)
