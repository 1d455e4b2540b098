"""GPU parity of the slot-indexed state pool (gdn_chunk_fwd_slots, gdn_recurrent_step_slots).

Expected values come from the fp64 oracle run on the states gathered from the
pool (zeros for padding sequences); the expected pool is the input pool with
the active rows replaced by the oracle's final states.  Rows no sequence names
must be left bit-identical.
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


def _slot_map(n_seq, n_slots, n_pad, seed):
    rng = np.random.default_rng(seed)
    ids = rng.permutation(n_slots)[:n_seq].astype(np.int32)
    pad = rng.choice(n_seq, size=n_pad, replace=False)
    ids[pad[: n_pad // 2]] = -1
    ids[pad[n_pad // 2:]] = n_slots + 3          # out of range: also padding
    return ids


def _expected_pool(pool, ids, final, n_slots):
    exp = pool.clone().double().numpy()
    for n, s in enumerate(ids):
        if 0 <= s < n_slots:
            exp[s] = final[n]
    return exp


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_decode_slots_against_oracle(io):
    from gated_deltanet_chunk_b200 import recurrent_step_slots
    N, P, steps = 64, 96, 6
    d = W.make_decode(num_seqs=N, steps=steps, nqk=4, nv=8, io=io, seed=51)
    ids = _slot_map(N, P, 6, 51)
    pool = torch.randn(P, 8, 128, 128, generator=torch.Generator().manual_seed(52)) * 0.1
    gpool, gids = pool.cuda(), torch.from_numpy(ids).cuda()
    outs = []
    for t in range(steps):
        outs.append(recurrent_step_slots(d["q"][t].cuda(), d["k"][t].cuda(), d["v"][t].cuda(),
                                         d["g"][t].cuda(), d["beta"][t].cuda(), gpool, gids))
    torch.cuda.synchronize()
    active = [n for n in range(N) if 0 <= ids[n] < P]
    pad = [n for n in range(N) if not 0 <= ids[n] < P]
    go = torch.stack(outs)                        # [steps, N, Nv, Dv]
    assert torch.count_nonzero(go[:, pad]) == 0   # padding rows: zero output
    pick = lambda x: x[:, active].transpose(0, 1).reshape(len(active) * steps, *x.shape[2:])
    s0 = pool[torch.as_tensor(ids[active].astype(np.int64))]
    cu = torch.arange(len(active) + 1, dtype=torch.int32) * steps
    ref_o, ref_s = oracle.recurrent(pick(d["q"]), pick(d["k"]), pick(d["v"]), pick(d["g"]),
                                    pick(d["beta"]), s0, cu)
    U.check_prefill(pick(go.cpu()), gpool[torch.as_tensor(ids[active].astype(np.int64))].cpu(),
                    ref_o, ref_s, cu, U.TOL[io], "decode-slots")
    untouched = sorted(set(range(P)) - set(int(ids[n]) for n in active))
    assert torch.equal(gpool[untouched].cpu(), pool[untouched])


@pytest.mark.parametrize("io,d,kernel", [("bf16", 128, "tc"), ("f32", 64, "auto")])
def test_multi_token_slots_against_oracle(io, d, kernel):
    """Per-sequence token counts 1..100 into a permuted pool: decode, multi-token steps, prefill."""
    from gated_deltanet_chunk_b200 import chunk_fwd_slots
    lens = [1, 2, 3, 5, 1, 64, 100, 4, 1, 17, 2, 3]
    N, P = len(lens), 20
    w = W.make_prefill(lengths=lens, nqk=2, nv=4, d=d, io=io, init_state=False, seed=53)
    ids = _slot_map(N, P, 2, 53)
    pool = torch.randn(P, 4, d, d, generator=torch.Generator().manual_seed(54)) * 0.1
    gpool = pool.cuda()
    out = chunk_fwd_slots(w["q"].cuda(), w["k"].cuda(), w["v"].cuda(), w["g"].cuda(), w["beta"].cuda(),
                          gpool, torch.from_numpy(ids).cuda(), w["cu_seqlens"].cuda(), chunk_size=64,
                          kernel=kernel)
    torch.cuda.synchronize()
    s0 = torch.zeros(N, 4, d, d)
    for n, s in enumerate(ids):
        if 0 <= s < P:
            s0[n] = pool[s]
    ref_o, ref_s = oracle.recurrent(w["q"], w["k"], w["v"], w["g"], w["beta"], s0, w["cu_seqlens"])
    assert U.rel_inf(U.to_np(out), ref_o) <= U.TOL[io]
    exp_pool = _expected_pool(pool, ids, ref_s, P)
    assert U.rel_inf(U.to_np(gpool), exp_pool) <= U.TOL[io]
    untouched = sorted(set(range(P)) - set(int(s) for s in ids if 0 <= s < P))
    assert torch.equal(gpool[untouched].cpu(), pool[untouched])


def test_identity_slots_equal_plain_decode():
    from gated_deltanet_chunk_b200 import recurrent_step, recurrent_step_slots
    d = W.make_decode(num_seqs=32, steps=1, nqk=4, nv=8, io="bf16", seed=55, device="cuda")
    st1, st2 = d["initial_state"].clone(), d["initial_state"].clone()
    ids = torch.arange(32, dtype=torch.int32, device="cuda")
    o1 = recurrent_step(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], st1)
    o2 = recurrent_step_slots(d["q"][0], d["k"][0], d["v"][0], d["g"][0], d["beta"][0], st2, ids)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(st1, st2)
