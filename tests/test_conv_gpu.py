"""GPU parity of the causal conv1d + SiLU that produces q, k, v (NEXT-3):
gdn_qkv_conv_fwd (prefill) and gdn_qkv_conv_update (decode).

Expected values: the fp64 oracle's causal_conv1d (walkthrough section 3 and its
torch_causal_conv1d_update) on the same stored inputs, split into the q | k | v
channel ranges.  The conv states hold copies of inputs, so they must match
bit for bit.  Bars on y: 1e-5 (fp32 io) and 1e-2 (bf16 io: one rounding of the
output), as max |x - y| / max |y| per output tensor.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import parity_utils as U

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    import gated_deltanet_chunk_b200 as g
    g.lib()


def _split(y, nqk, nv, dk, dv):
    qk = nqk * dk
    T = y.shape[0]
    return (y[:, :qk].reshape(T, nqk, dk), y[:, qk:2 * qk].reshape(T, nqk, dk),
            y[:, 2 * qk:].reshape(T, nv, dv))


def _check(gq, gk, gv, ref, io, nqk, nv, dk, dv, what):
    for name, g_, r_ in zip("qkv", (gq, gk, gv), _split(ref, nqk, nv, dk, dv)):
        e = U.rel_inf(U.to_np(g_), r_)
        assert e <= TOL[io], (what, name, e)


@pytest.mark.parametrize("io,K,with_state,with_bias", [("bf16", 4, True, True), ("bf16", 4, False, True),
                                                      ("f32", 4, True, False), ("f32", 2, True, True),
                                                      ("bf16", 1, False, False), ("bf16", 3, True, True)])
def test_conv_fwd_against_oracle(io, K, with_state, with_bias):
    from gated_deltanet_chunk_b200 import qkv_conv_fwd
    nqk, nv, dk, dv = 2, 4, 64, 128
    lens = [1, 2, 3, 5, 64, 0, 300, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    c = W.make_conv_inputs(T, nqk, nv, dk, dv, K, io, seed=71 + K, num_states=len(lens) if with_state else 0,
                           bias=with_bias)
    d = lambda t: None if t is None else t.cuda()
    q, k, v, st = qkv_conv_fwd(d(c["x"]), d(c["weight"]), nqk, nv, dk, dv, bias=d(c["bias"]),
                               conv_state=d(c["state"]), cu_seqlens=torch.from_numpy(cu).cuda())
    torch.cuda.synchronize()
    ref_y, ref_s = oracle.causal_conv1d(c["x"], c["weight"], c["bias"], cu, c["state"])
    _check(q, k, v, ref_y, io, nqk, nv, dk, dv, "fwd")
    assert np.array_equal(U.to_np(st), ref_s)


def test_conv_fwd_in_place_state_and_equal_lengths():
    from gated_deltanet_chunk_b200 import qkv_conv_fwd
    nqk, nv, dk, dv, K = 1, 2, 128, 64, 4
    c = W.make_conv_inputs(3 * 129, nqk, nv, dk, dv, K, "bf16", seed=72, num_states=3)
    st = c["state"].cuda()
    q, k, v, out_state = qkv_conv_fwd(c["x"].cuda(), c["weight"].cuda(), nqk, nv, dk, dv, bias=c["bias"].cuda(),
                                      conv_state=st, num_seqs=3, state_out=st)
    torch.cuda.synchronize()
    cu = np.arange(4, dtype=np.int32) * 129
    ref_y, ref_s = oracle.causal_conv1d(c["x"], c["weight"], c["bias"], cu, c["state"])
    _check(q, k, v, ref_y, "bf16", nqk, nv, dk, dv, "in-place")
    assert out_state.data_ptr() == st.data_ptr()
    assert np.array_equal(U.to_np(st), ref_s)


@pytest.mark.parametrize("K", [1, 2, 3, 4])
@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_conv_update_equals_prefill_and_oracle(io, K):
    """Per-token decode updates = one prefill over the same tokens; slot pool with padding rows.
    N = 17 leaves a ragged last group of the sequences a thread takes (4)."""
    from gated_deltanet_chunk_b200 import qkv_conv_fwd, qkv_conv_update
    nqk, nv, dk, dv, N, steps, P = 2, 4, 128, 128, 17, 7, 40
    c = W.make_conv_inputs(N * steps, nqk, nv, dk, dv, K, io, seed=73, num_states=P)
    x = c["x"].reshape(steps, N, c["C"])                    # token t of sequence n at x[t, n]
    ids = np.random.default_rng(73).permutation(P)[:N].astype(np.int32)
    ids[[3, 11]] = [-1, P + 5]                              # two padding sequences
    pool = c["state"].cuda()
    gids = torch.from_numpy(ids).cuda()
    outs = []
    for t in range(steps):
        outs.append(qkv_conv_update(x[t].cuda().contiguous(), c["weight"].cuda(), pool, nqk, nv, dk, dv,
                                    bias=c["bias"].cuda(), slot_ids=gids))
    torch.cuda.synchronize()
    active = [n for n in range(N) if 0 <= ids[n] < P]
    # oracle: sequence n = its tokens x[:, n] after the window pool[ids[n]]
    seqs = x[:, active].transpose(0, 1).reshape(len(active) * steps, c["C"])
    cu = np.arange(len(active) + 1, dtype=np.int32) * steps
    s0 = c["state"][torch.as_tensor(ids[active].astype(np.int64))]
    ref_y, ref_s = oracle.causal_conv1d(seqs, c["weight"], c["bias"], cu, s0)
    ref_y = ref_y.reshape(len(active), steps, c["C"])
    for t in range(steps):
        q, k, v = outs[t]
        for n in (3, 11):
            assert torch.count_nonzero(q[n]) == 0 and torch.count_nonzero(v[n]) == 0
        _check(q[active], k[active], v[active], ref_y[:, t], io, nqk, nv, dk, dv, "update step %d" % t)
    gp = U.to_np(pool)
    assert np.array_equal(gp[ids[active]], ref_s)
    untouched = [s for s in range(P) if s not in ids[active]]
    assert np.array_equal(gp[untouched], U.to_np(c["state"])[untouched])
    # the same tokens as one prefill per sequence give the same q, k, v
    q2, k2, v2, st2 = qkv_conv_fwd(seqs.cuda().contiguous(), c["weight"].cuda(), nqk, nv, dk, dv,
                                   bias=c["bias"].cuda(), conv_state=s0.cuda().contiguous(),
                                   cu_seqlens=torch.from_numpy(cu).cuda())
    torch.cuda.synchronize()
    qa = torch.stack([outs[t][0][active] for t in range(steps)], 1).reshape(len(active) * steps, nqk, dk)
    assert torch.equal(qa, q2)
    assert np.array_equal(U.to_np(st2), ref_s)


def test_conv_fwd_full_size_sampled_channels():
    """The long prefill's shape (2 x 32768 tokens, C = 8192): 48 channels from every range
    checked against the oracle (channels are independent)."""
    from gated_deltanet_chunk_b200 import qkv_conv_fwd
    nqk, nv, dk, dv, K, n, L = 16, 32, 128, 128, 4, 2, 32768
    c = W.make_conv_inputs(n * L, nqk, nv, dk, dv, K, "bf16", seed=74)
    q, k, v, st = qkv_conv_fwd(c["x"].cuda(), c["weight"].cuda(), nqk, nv, dk, dv, bias=c["bias"].cuda(),
                               num_seqs=n)
    torch.cuda.synchronize()
    y = torch.cat([q.reshape(n * L, -1), k.reshape(n * L, -1), v.reshape(n * L, -1)], 1)
    chans = np.concatenate([np.arange(0, 16), np.arange(2040, 2056), np.arange(8176, 8192)])
    cu = np.array([0, L, 2 * L], dtype=np.int32)
    ref_y, ref_s = oracle.causal_conv1d(c["x"][:, chans], c["weight"][chans], c["bias"][chans], cu, None)
    assert U.rel_inf(U.to_np(y[:, chans]), ref_y) <= TOL["bf16"]
    assert np.array_equal(U.to_np(st[:, chans]), ref_s)


def _fused_decode_case(io, nqk, nv, N, steps, P, pad, seed):
    dk = dv = 128
    c = W.make_conv_inputs(N * steps, nqk, nv, dk, dv, 4, io, seed=seed, num_states=P)
    d = W.make_decode(num_seqs=N, steps=steps, nqk=nqk, nv=nv, io=io, seed=seed)
    ids = np.random.default_rng(seed).permutation(P)[:N].astype(np.int32)
    for n in pad:
        ids[n] = -1
    pool = torch.randn(P, nv, dk, dv, generator=torch.Generator().manual_seed(seed)) * 0.1
    return c, d, ids, pool


def _oracle_fused_decode(c, d, ids, pool, nqk, nv, N, steps, P, gates=None, norm=None):
    """Conv over each sequence's tokens after its cached window, then the token recurrence."""
    dk = dv = 128
    active = [n for n in range(N) if 0 <= ids[n] < P]
    x = c["x"].reshape(steps, N, c["C"])
    seqs = x[:, active].transpose(0, 1).reshape(len(active) * steps, c["C"])
    cu = np.arange(len(active) + 1, dtype=np.int32) * steps
    idx = torch.as_tensor(ids[active].astype(np.int64))
    y, cs = oracle.causal_conv1d(seqs, c["weight"], c["bias"], cu, c["state"][idx])
    q, k, v = _split(y, nqk, nv, dk, dv)
    pick = lambda t: t[:, active].transpose(0, 1).reshape(len(active) * steps, *t.shape[2:])
    g, beta = (pick(d["g"]), pick(d["beta"])) if gates is None else gates(pick)
    o, sf = oracle.recurrent(q, k, v, g, beta, pool[idx], cu)
    if norm is not None:
        o = oracle.gated_rmsnorm(o, pick(norm[0]), norm[1], 1e-6)
    return active, o.reshape(len(active), steps, nv, dv), sf, cs


@pytest.mark.parametrize("io,nqk,nv", [("bf16", 2, 4), ("f32", 4, 4), ("bf16", 1, 8)])
def test_decode_with_fused_conv_against_oracle(io, nqk, nv):
    from gated_deltanet_chunk_b200 import recurrent_step_ex
    N, steps, P = 24, 5, 40
    c, d, ids, pool = _fused_decode_case(io, nqk, nv, N, steps, P, pad=[5], seed=81 + nv)
    gpool, gcs, gids = pool.cuda(), c["state"].cuda(), torch.from_numpy(ids).cuda()
    x = c["x"].reshape(steps, N, c["C"]).cuda()
    outs = []
    for t in range(steps):
        outs.append(recurrent_step_ex(None, None, None, d["g"][t].cuda(), d["beta"][t].cuda(), gpool,
                                      slot_ids=gids, conv_x=x[t], conv_state=gcs, conv_weight=c["weight"].cuda(),
                                      conv_bias=c["bias"].cuda(), shapes=(nqk, nv, 128, 128)))
    torch.cuda.synchronize()
    active, ref_o, ref_s, ref_cs = _oracle_fused_decode(c, d, ids, pool, nqk, nv, N, steps, P)
    go = torch.stack(outs, 1)                                  # [N, steps, Nv, Dv]
    assert torch.count_nonzero(go[5]) == 0                     # padding row
    tol = U.TOL[io]
    for i, n in enumerate(active):
        assert U.rel_inf(U.to_np(go[n]), ref_o[i]) <= tol, n
    idx = torch.as_tensor(ids[active].astype(np.int64))
    assert U.rel_inf(U.to_np(gpool[idx]), ref_s) <= tol
    assert np.array_equal(U.to_np(gcs[idx]), ref_cs)           # conv windows: copies of inputs
    untouched = [s for s in range(P) if s not in ids[active]]
    assert torch.equal(gcs[untouched].cpu(), c["state"][untouched])


def test_fused_conv_equals_two_launches_and_all_fusions():
    """The fused step leaves the same conv state as gdn_qkv_conv_update + gdn_recurrent_step and
    outputs within the bf16 rounding of q, k, v the two-launch path adds; then gate + slots +
    norm + conv together against the oracle."""
    from gated_deltanet_chunk_b200 import qkv_conv_update, recurrent_step, recurrent_step_ex
    nqk, nv, N, steps, P = 2, 4, 16, 4, 16
    c, d, ids, pool = _fused_decode_case("bf16", nqk, nv, N, steps, P, pad=[], seed=91)
    ids = np.arange(N, dtype=np.int32)                         # plain rows
    x = c["x"].reshape(steps, N, c["C"]).cuda()
    w, b = c["weight"].cuda(), c["bias"].cuda()
    s1, cs1 = pool.cuda(), c["state"].cuda()
    s2, cs2 = pool.cuda(), c["state"].cuda()
    for t in range(steps):
        o1 = recurrent_step_ex(None, None, None, d["g"][t].cuda(), d["beta"][t].cuda(), s1, conv_x=x[t],
                               conv_state=cs1, conv_weight=w, conv_bias=b, shapes=(nqk, nv, 128, 128))
        q, k, v = qkv_conv_update(x[t], w, cs2, nqk, nv, 128, 128, bias=b)
        o2 = recurrent_step(q, k, v, d["g"][t].cuda(), d["beta"][t].cuda(), s2)
        torch.cuda.synchronize()
        assert U.rel_inf(U.to_np(o1), U.to_np(o2)) < 2e-2
    assert torch.equal(cs1, cs2)
    # everything at once
    z, nw = W.make_norm_inputs(d["v"].shape, "bf16", seed=92)
    s3, cs3 = pool.cuda(), c["state"].cuda()
    gids = torch.from_numpy(ids).cuda()
    outs = []
    for t in range(steps):
        outs.append(recurrent_step_ex(None, None, None, d["a"][t].cuda(), d["b"][t].cuda(), s3,
                                      A_log=d["A_log"].cuda(), dt_bias=d["dt_bias"].cuda(), slot_ids=gids,
                                      norm_z=z[t].cuda(), norm_weight=nw.cuda(), conv_x=x[t], conv_state=cs3,
                                      conv_weight=w, conv_bias=b, shapes=(nqk, nv, 128, 128)))
    torch.cuda.synchronize()
    gates = lambda pick: oracle.gates(pick(d["a"]), pick(d["b"]), d["A_log"], d["dt_bias"])
    active, ref_o, ref_s, ref_cs = _oracle_fused_decode(c, d, ids, pool, nqk, nv, N, steps, P, gates=gates,
                                                        norm=(z, nw))
    go = torch.stack(outs, 1)
    for i, n in enumerate(active):
        assert U.rel_inf(U.to_np(go[n]), ref_o[i]) <= U.TOL["bf16"], n
    assert U.rel_inf(U.to_np(s3), ref_s) <= U.TOL["bf16"]
    assert np.array_equal(U.to_np(cs3), ref_cs)


def test_conv_fwd_empty_batch_keeps_the_windows():
    """total_tokens = 0: no q, k, v rows; the new conv_state is the old window, bit for bit."""
    from gated_deltanet_chunk_b200 import qkv_conv_fwd
    c = W.make_conv_inputs(0, 2, 4, 64, 128, 4, "bf16", seed=97, num_states=3)
    q, k, v, st = qkv_conv_fwd(c["x"].cuda(), c["weight"].cuda(), 2, 4, 64, 128, bias=c["bias"].cuda(),
                               conv_state=c["state"].cuda(), cu_seqlens=torch.zeros(4, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert q.numel() == 0 and v.numel() == 0
    assert torch.equal(st.cpu(), c["state"])


def test_fused_conv_norm_decode_full_shape_sampled():
    """The decode workload's shape (256 sequences, Nqk 16, Nv 32, D 128) with the conv and the
    norm fused into the step, 3 steps; 8 sequences checked against the oracle (all heads)."""
    from gated_deltanet_chunk_b200 import recurrent_step_ex
    N, nqk, nv, steps = 256, 16, 32, 3
    d = W.make_decode(num_seqs=N, steps=steps, nqk=nqk, nv=nv, io="bf16", seed=98)
    c = W.make_conv_inputs(N * steps, nqk, nv, 128, 128, 4, "bf16", seed=98, num_states=N)
    z, nw = W.make_norm_inputs(d["v"].shape, "bf16", seed=98)
    x = c["x"].reshape(steps, N, c["C"]).cuda()
    state, cst = d["initial_state"].cuda(), c["state"].cuda()
    outs = []
    for t in range(steps):
        outs.append(recurrent_step_ex(None, None, None, d["g"][t].cuda(), d["beta"][t].cuda(), state,
                                      norm_z=z[t].cuda(), norm_weight=nw.cuda(), conv_x=x[t], conv_state=cst,
                                      conv_weight=c["weight"].cuda(), conv_bias=c["bias"].cuda(),
                                      shapes=(nqk, nv, 128, 128)))
    torch.cuda.synchronize()
    pick_seqs = [0, 1, 37, 100, 128, 199, 254, 255]
    idx = torch.as_tensor(pick_seqs)
    xs = c["x"].reshape(steps, N, c["C"])[:, idx].transpose(0, 1).reshape(len(idx) * steps, c["C"])
    cu = np.arange(len(idx) + 1, dtype=np.int32) * steps
    y, ref_cs = oracle.causal_conv1d(xs, c["weight"], c["bias"], cu, c["state"][idx])
    q, k, v = _split(y, nqk, nv, 128, 128)
    pick = lambda t: t[:, idx].transpose(0, 1).reshape(len(idx) * steps, *t.shape[2:])
    o, sf = oracle.recurrent(q, k, v, pick(d["g"]), pick(d["beta"]), d["initial_state"][idx], cu)
    o = oracle.gated_rmsnorm(o, pick(z), nw, 1e-6).reshape(len(idx), steps, nv, 128)
    go = torch.stack(outs, 1)[idx]
    for i in range(len(idx)):
        assert U.rel_inf(U.to_np(go[i]), o[i]) <= U.TOL["bf16"], pick_seqs[i]
    assert U.rel_inf(U.to_np(state[idx.cuda()]), sf) <= U.TOL["bf16"]
    assert np.array_equal(U.to_np(cst[idx.cuda()]), ref_cs)


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_silu_evaluation_error_bound(io):
    """With the last tap 1, the others 0, no bias and an empty window, the conv is silu(x) itself.
    Per element against x sigmoid(x) in fp64, over x in [-20, 20], in both the prefill and the
    update kernels: bf16 outputs within their rounding (2^-8 relative) plus |x| 2^-12 (SiLU as
    h + h tanh(h), h = x / 2, with tanh.approx's 2^-11 relative bound); fp32 outputs within
    1e-5 relative (the exp / divide intrinsics)."""
    from gated_deltanet_chunk_b200 import qkv_conv_fwd, qkv_conv_update
    nqk, nv, d, K, T = 1, 1, 128, 4, 64
    C = 2 * nqk * d + nv * d
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    x = torch.linspace(-20.0, 20.0, T * C, dtype=torch.float64).reshape(T, C).to(dt)
    w = torch.zeros(C, K, dtype=torch.float32)
    w[:, K - 1] = 1.0
    xd = x.double().numpy()
    ref = xd / (1.0 + np.exp(-xd))
    if io == "bf16":
        bound = 2.0 ** -8 * np.abs(ref) + 1.01 * 2.0 ** -12 * np.abs(xd) + 1e-30
    else:
        bound = 1e-5 * np.abs(ref) + 1e-30
    q, k, v, _ = qkv_conv_fwd(x.cuda(), w.cuda(), nqk, nv, d, d, num_seqs=1, output_state=False)
    state = torch.zeros(T, C, K, dtype=dt, device="cuda")
    q2, k2, v2 = qkv_conv_update(x.cuda(), w.cuda(), state, nqk, nv, d, d)
    torch.cuda.synchronize()
    for what, parts in (("prefill", (q, k, v)), ("update", (q2, k2, v2))):
        y = torch.cat([p_.reshape(T, -1) for p_ in parts], 1).double().cpu().numpy()
        err = np.abs(y - ref)
        worst = int(np.argmax(err / bound))
        assert np.all(err <= bound), (what, float(xd.flat[worst]), float(y.flat[worst]), float(ref.flat[worst]))
