"""Device-side checks of the data preconditions, tested without a GPU fault.

cu_seqlens must be non-decreasing from 0 to total_tokens (the packed layout of
the PyPTO-Gym "Qwen3Next 样例" README, 参数说明: act_seq_len), and the
tensor-core chunk kernel needs every gate g <= 0 (the layer's gate
-exp(A_log) softplus(a + dt_bias) of the "手撕Qwen3-Next" walkthrough,
section 一(一)4, always is).  The kernels clamp every sequence's bounds into
[0, total_tokens], so an inconsistent cu_seqlens leads to no access outside the
tensors; they report it (GDN_ERR_SEQLENS) and a gate g > 0 (GDN_ERR_GATE)
through the status word that gdn_device_status reads and clears.  After each
bad call a clean call still matches the oracle and reports GDN_OK.
"""
import pytest
import torch

import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu

GDN_ERR_SEQLENS, GDN_ERR_GATE = -8, -9


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()
    g.device_status()  # start from a clear word


def _clean_prefill_matches(kernel):
    import gated_deltanet_chunk_b200 as g
    w = W.make_prefill(lengths=[130, 7, 64], nqk=1, nv=2, d=128, io="bf16", init_state=True, seed=97)
    out, sf = U.run_gpu_prefill(w, 64, kernel)
    ref_o, ref_s = U.run_oracle_prefill(w)
    U.check_prefill(out, sf, ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"], "clean-after-" + kernel)
    assert g.device_status() == 0


# cu_seqlens for T = 300 tokens: out of order; last entry short of T; beyond T; first entry not 0
BAD_CU = {"decreasing": [0, 200, 100, 300], "short": [0, 100, 250], "beyond": [0, 100, 900],
          "nonzero_start": [40, 100, 300]}


@pytest.mark.parametrize("case", sorted(BAD_CU))
@pytest.mark.parametrize("kernel", ["tc", "simt"])
def test_inconsistent_cu_seqlens_reported_not_faulted(case, kernel):
    import gated_deltanet_chunk_b200 as g
    cu = BAD_CU[case]
    T = 300
    w = W.make_prefill(num_seqs=1, seq_len=T, nqk=1, nv=2, d=128, io="bf16", init_state=False, seed=98)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    cus = torch.tensor(cu, dtype=torch.int32, device="cuda")
    out, sf = g.chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], None, cus, chunk_size=64, kernel=kernel)
    torch.cuda.synchronize()
    assert g.device_status() == GDN_ERR_SEQLENS
    assert g.device_status() == 0  # the read cleared it
    _clean_prefill_matches(kernel)


@pytest.mark.parametrize("case", sorted(BAD_CU))
def test_inconsistent_cu_seqlens_conv_reported(case):
    import gated_deltanet_chunk_b200 as g
    cu = torch.tensor(BAD_CU[case], dtype=torch.int32, device="cuda")
    T, nqk, nv, D = 300, 1, 2, 128
    cv = W.make_conv_inputs(T, nqk, nv, D, D, 4, "bf16", seed=99, num_states=cu.numel() - 1, device="cuda")
    st = torch.empty_like(cv["state"])
    g.qkv_conv_fwd(cv["x"], cv["weight"], nqk, nv, D, D, bias=cv["bias"], conv_state=cv["state"],
                   cu_seqlens=cu, state_out=st)
    torch.cuda.synchronize()
    assert g.device_status() == GDN_ERR_SEQLENS
    assert g.device_status() == 0


def test_positive_gate_reported_by_tensor_core_kernel():
    import gated_deltanet_chunk_b200 as g
    w = W.make_prefill(lengths=[200, 90], nqk=1, nv=2, d=128, io="bf16", init_state=True, seed=100)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in w.items()}
    gpos = d["g"].clone()
    gpos[150, 1] = 0.5  # one gate of sequence 0, v-head 1, is positive
    g.chunk_fwd(d["q"], d["k"], d["v"], gpos, d["beta"], d["initial_state"], d["cu_seqlens"], chunk_size=64,
                kernel="tc")
    torch.cuda.synchronize()
    assert g.device_status() == GDN_ERR_GATE
    assert g.device_status() == 0
    # the CUDA-core kernel takes any finite gate and reports nothing
    out, sf = g.chunk_fwd(d["q"], d["k"], d["v"], gpos, d["beta"], d["initial_state"], d["cu_seqlens"],
                          chunk_size=64, kernel="simt")
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ref_o, ref_s = oracle_prefill_with_gate(w, gpos.cpu())
    U.check_prefill(out, sf, ref_o, ref_s, w["cu_seqlens"], U.TOL["bf16"], "positive-gate-simt")
    _clean_prefill_matches("tc")


def oracle_prefill_with_gate(w, gate):
    w2 = dict(w)
    w2["g"] = gate
    return U.run_oracle_prefill(w2)
