"""The seeded input generators: shapes, determinism and the varlen recipe (no GPU)."""
import torch

import workloads as W


def test_prefill_shapes_and_determinism():
    a = W.make_prefill(num_seqs=3, seq_len=50, nqk=2, nv=4, d=16, io="bf16", init_state=True, seed=5)
    b = W.make_prefill(num_seqs=3, seq_len=50, nqk=2, nv=4, d=16, io="bf16", init_state=True, seed=5)
    assert a["q"].shape == (150, 2, 16) and a["q"].dtype == torch.bfloat16
    assert a["v"].shape == (150, 4, 16)
    assert a["g"].shape == (150, 4) and a["g"].dtype == torch.float32
    assert a["initial_state"].shape == (3, 4, 16, 16)
    assert a["cu_seqlens"].tolist() == [0, 50, 100, 150]
    for key in ("q", "k", "v", "g", "beta", "initial_state"):
        assert torch.equal(a[key], b[key])
    assert bool((a["g"] < 0).all()) and bool(((a["beta"] > 0) & (a["beta"] < 1)).all())


def test_varlen_recipe():
    gen = torch.Generator().manual_seed(3)
    lens = W.varlen_lengths(32, 100, 16384, gen, 64)
    assert int(lens.min()) >= 100 and int(lens.max()) <= 16384
    assert bool(((lens % 64) == 1).any())
    w = W.make_workload("tiny_f32_d64", seed=0)
    assert w["T"] == 256 and w["chunk"] == 64 and w["initial_state"] is None


def test_gate_modes():
    z = W.make_prefill(seq_len=20, gate="zero_beta1")
    assert bool((z["g"] == 0).all()) and bool((z["beta"] == 1).all())
    d = W.make_decode(num_seqs=4, steps=3, nqk=2, nv=4, d=16)
    assert d["q"].shape == (3, 4, 2, 16) and d["initial_state"].shape == (4, 4, 16, 16)
