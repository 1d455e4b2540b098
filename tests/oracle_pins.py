"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

Each ``pin_*`` function raises AssertionError on failure.  They are collected
by ``test_oracle.py`` and re-run against deliberately broken builds of the
oracle by ``test_oracle_mutants.py`` (every mutant must fail at least one pin).

Sources: the "手撕Qwen3-Next" walkthrough (section 5(1) chunkwise recurrence,
section 5(2) token recurrence and its DeltaNet derivation, section 4 GQA
repeat) and the PyPTO-Gym "Qwen3Next 样例" README (数学公式: L2 norm with eps
inside the root; 参数说明: packed tensors with cumulative lengths).
"""
from __future__ import annotations

import numpy as np

import oracle

TOL = 1e-10  # fp64 agreement between algebraically identical forms


def rel(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return float(np.max(np.abs(x - y)) / max(float(np.max(np.abs(y))), 1e-30))


def rand_case(rng, T=24, nqk=1, nv=1, dk=8, dv=6, s0=True, gate="mild", lengths=None):
    """Small fp64 case; ``gate``: "mild" (A ~ U(0,1)), "layer" (A ~ U(0,16)), "zero"."""
    if lengths is not None:
        T = int(sum(lengths))
    q = rng.standard_normal((T, nqk, dk))
    k = rng.standard_normal((T, nqk, dk))
    v = rng.standard_normal((T, nv, dv))
    b = rng.standard_normal((T, nv))
    a = rng.standard_normal((T, nv))
    A = rng.uniform(0, 1.0 if gate == "mild" else 16.0, size=nv)
    g = -A * np.log1p(np.exp(a + 1.0))
    if gate == "zero":
        g = np.zeros_like(g)
    beta = 1.0 / (1.0 + np.exp(-b))
    n = 1 if lengths is None else len(lengths)
    cu = np.array([0, T], dtype=np.int32) if lengths is None else \
        np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    S0 = 0.5 * rng.standard_normal((n, nv, dk, dv)) if s0 else None
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=S0, cu_seqlens=cu)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# (i) the code form of the token update equals the DeltaNet matrix form
#     S_t = S_{t-1}(alpha_t (I - beta_t k k^T)) + beta_t v k^T   ([dv, dk] on the
#     page; here transposed to the [dk, dv] storage), o_t = S_t^T q.
#     Non-symmetric S0 and Dk != Dv pin the storage orientation.
# --------------------------------------------------------------------------
def pin_matrix_form():
    rng = np.random.default_rng(1)
    c = rand_case(rng, T=30, dk=8, dv=6)
    dk = 8
    out, sf = oracle.recurrent(**c)
    qn = c["q"][:, 0] / np.sqrt((c["q"][:, 0] ** 2).sum(-1, keepdims=True) + 1e-6) / np.sqrt(dk)
    kn = c["k"][:, 0] / np.sqrt((c["k"][:, 0] ** 2).sum(-1, keepdims=True) + 1e-6)
    S = c["initial_state"][0, 0].copy()
    ref = np.zeros_like(out)
    for t in range(30):
        al, be, kk, vv = np.exp(c["g"][t, 0]), c["beta"][t, 0], kn[t], c["v"][t, 0]
        St = S.T  # [dv, dk] orientation of the page
        St = St @ (al * (np.eye(dk) - be * np.outer(kk, kk))) + be * np.outer(vv, kk)
        S = St.T
        ref[t, 0] = S.T @ qn[t]
    assert rel(out, ref) < TOL, rel(out, ref)
    assert rel(sf[0, 0], S) < TOL


# --------------------------------------------------------------------------
# L2 norm of the PyPTO README: x / sqrt(sum x^2 + eps), eps = 1e-6 inside the
# root.  One token, S0 = 0, g = 0, beta = 1, q = k = a tiny vector x:
#   o = (q_hat . k_hat) v = scale * |x|^2 / (|x|^2 + eps) * v.
# --------------------------------------------------------------------------
def pin_l2norm_eps_closed_form():
    dk, dv = 4, 3
    x = np.array([1e-4, -2e-4, 0.5e-4, 1e-4]).reshape(1, 1, dk)
    v = np.array([1.0, -2.0, 3.0]).reshape(1, 1, dv)
    g = np.zeros((1, 1))
    beta = np.ones((1, 1))
    out, _ = oracle.recurrent(x, x, v, g, beta)
    n2 = float((x ** 2).sum())
    ref = (1.0 / np.sqrt(dk)) * n2 / (n2 + 1e-6) * v
    assert rel(out, ref) < TOL, (out, ref)


# --------------------------------------------------------------------------
# The norm makes q and k scale-free, and the query scale is 1/sqrt(Dk) by
# default (walkthrough 5(1)a); an explicit scale multiplies the output.
# --------------------------------------------------------------------------
def pin_scale_and_norm_invariance():
    rng = np.random.default_rng(2)
    c = rand_case(rng, T=20, dk=16, dv=5)
    o1, s1 = oracle.recurrent(**c)
    c2 = dict(c, q=c["q"] * 37.0, k=c["k"] * 53.0)
    o2, s2 = oracle.recurrent(**c2)
    assert rel(o2, o1) < 1e-6 and rel(s2, s1) < 1e-6  # eps/|x|^2 effects only (~6e-8 here)
    o3, _ = oracle.recurrent(**c, scale=1.0 / np.sqrt(16.0))
    assert rel(o3, o1) < TOL
    o4, _ = oracle.recurrent(**c, scale=0.5)
    assert rel(o4, o1 * 0.5 * np.sqrt(16.0)) < TOL


# --------------------------------------------------------------------------
# (ii) the chunk closed form equals the token recurrence for every chunk size
#      (walkthrough 5(1) vs 5(2)); padded tails, GQA, random S0.
# --------------------------------------------------------------------------
def pin_chunk_equals_recurrent():
    rng = np.random.default_rng(3)
    for (T, dk, dv, nqk, nv, Cs, gate) in [
        (37, 4, 4, 1, 1, (1, 2, 4, 16, 64), "mild"),
        (130, 16, 12, 1, 2, (16, 64, 128), "mild"),
        (150, 64, 64, 2, 4, (64, 128), "layer"),
        (70, 128, 128, 1, 1, (64,), "zero"),
    ]:
        c = rand_case(rng, T=T, nqk=nqk, nv=nv, dk=dk, dv=dv, gate=gate)
        o_ref, s_ref = oracle.recurrent(**c)
        for C in Cs:
            o, s = oracle.chunk_form(**c, chunk_size=C)
            assert rel(o, o_ref) < TOL, (T, dk, C, rel(o, o_ref))
            assert rel(s, s_ref) < TOL, (T, dk, C, rel(s, s_ref))


# --------------------------------------------------------------------------
# (iii) beta = 0: no writes.  S_T = S0 exp(sum g), o_t = q_hat^T S0 exp(sum_{s<=t} g_s).
# --------------------------------------------------------------------------
def pin_beta_zero():
    rng = np.random.default_rng(4)
    c = rand_case(rng, T=25, dk=8, dv=6)
    c["beta"] = np.zeros_like(c["beta"])
    for form in ("rec", "chunk"):
        if form == "rec":
            out, sf = oracle.recurrent(**c)
        else:
            out, sf = oracle.chunk_form(**c, chunk_size=8)
        G = np.cumsum(c["g"][:, 0])
        qn = c["q"][:, 0] / np.sqrt((c["q"][:, 0] ** 2).sum(-1, keepdims=True) + 1e-6) / np.sqrt(8)
        ref = np.exp(G)[:, None] * (qn @ c["initial_state"][0, 0])
        assert rel(out[:, 0], ref) < TOL, form
        assert rel(sf[0, 0], c["initial_state"][0, 0] * np.exp(G[-1])) < TOL, form


# --------------------------------------------------------------------------
# (iv) g = 0, beta = 1, unit keys: the delta rule writes v exactly, so
#      k_t^T S_t = v_t (walkthrough 5(2), DeltaNet derivation).
# --------------------------------------------------------------------------
def pin_delta_write_exact():
    rng = np.random.default_rng(5)
    T, dk, dv = 12, 8, 5
    c = rand_case(rng, T=T, dk=dk, dv=dv, gate="zero")
    c["beta"] = np.ones_like(c["beta"])
    c["k"] = unit_rows(c["k"])
    for t_end in range(1, T + 1):
        sub = dict(c, q=c["q"][:t_end], k=c["k"][:t_end], v=c["v"][:t_end], g=c["g"][:t_end],
                   beta=c["beta"][:t_end], cu_seqlens=np.array([0, t_end], dtype=np.int32))
        _, sf = oracle.recurrent(**sub, qk_l2norm=False)
        kv = c["k"][t_end - 1, 0] @ sf[0, 0]
        assert rel(kv, c["v"][t_end - 1, 0]) < 1e-12
    # with the in-kernel norm (eps 1e-6) the write is exact up to eps/|k|^2
    _, sf = oracle.recurrent(**dict(c, k=c["k"] * 3.0))
    assert rel(c["k"][-1, 0] @ sf[0, 0], c["v"][-1, 0]) < 1e-6


# --------------------------------------------------------------------------
# (v) chunk-size invariance and zero-pad invariance.
# --------------------------------------------------------------------------
def pin_zero_pad_invariance():
    rng = np.random.default_rng(6)
    c = rand_case(rng, T=21, dk=8, dv=6)
    o, s = oracle.recurrent(**c)
    pad = 11
    cp = {key: (np.concatenate([c[key], np.zeros((pad,) + c[key].shape[1:])]) if key in
                ("q", "k", "v", "g", "beta") else c[key]) for key in c}
    cp["cu_seqlens"] = np.array([0, 21 + pad], dtype=np.int32)
    op, sp = oracle.recurrent(**cp)
    assert rel(sp, s) < TOL and rel(op[:21], o) < TOL
    for C in (8, 16):
        oc, sc = oracle.chunk_form(**c, chunk_size=C)
        assert rel(sc, s) < TOL and rel(oc, o) < TOL


# --------------------------------------------------------------------------
# (vi) split and carry; varlen equals separate per-sequence calls, and every
#      sequence starts from its own initial state (PyPTO act_seq_len).
# --------------------------------------------------------------------------
def pin_split_carry_and_varlen():
    rng = np.random.default_rng(7)
    c = rand_case(rng, T=40, nqk=1, nv=2, dk=8, dv=6)
    o, s = oracle.recurrent(**c)
    for t in (1, 16, 23, 39):
        a = {key: (c[key][:t] if key in ("q", "k", "v", "g", "beta") else c[key]) for key in c}
        a["cu_seqlens"] = np.array([0, t], dtype=np.int32)
        oa, sa = oracle.recurrent(**a)
        b = {key: (c[key][t:] if key in ("q", "k", "v", "g", "beta") else c[key]) for key in c}
        b["cu_seqlens"] = np.array([0, 40 - t], dtype=np.int32)
        b["initial_state"] = sa
        ob, sb = oracle.recurrent(**b)
        assert rel(np.concatenate([oa, ob]), o) < TOL and rel(sb, s) < TOL, t
    lens = [5, 1, 17, 9]
    cv = rand_case(rng, nqk=1, nv=2, dk=8, dv=6, lengths=lens)
    ov, sv = oracle.recurrent(**cv)
    oc, sc = oracle.chunk_form(**cv, chunk_size=4)
    assert rel(oc, ov) < TOL and rel(sc, sv) < TOL
    cu = cv["cu_seqlens"]
    for n in range(len(lens)):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        one = {key: cv[key][sl] for key in ("q", "k", "v", "g", "beta")}
        on, sn = oracle.recurrent(**one, initial_state=cv["initial_state"][n:n + 1])
        assert rel(on, ov[sl]) < TOL and rel(sn[0], sv[n]) < TOL, n


# --------------------------------------------------------------------------
# (vii) GQA: v-head h reads qk-head floor(h / G), i.e. repeat_interleave
#       (walkthrough section 4).
# --------------------------------------------------------------------------
def pin_gqa_repeat_interleave():
    rng = np.random.default_rng(8)
    c = rand_case(rng, T=19, nqk=2, nv=6, dk=8, dv=4)
    o, s = oracle.recurrent(**c)
    rep = dict(c, q=np.repeat(c["q"], 3, axis=1), k=np.repeat(c["k"], 3, axis=1))
    o2, s2 = oracle.recurrent(**rep)
    assert rel(o, o2) < TOL and rel(s, s2) < TOL
    oc, sc = oracle.chunk_form(**c, chunk_size=4)
    assert rel(oc, o2) < TOL and rel(sc, s2) < TOL


# --------------------------------------------------------------------------
# (viii) linearity in (v, S0) jointly: T, W, gamma and gcum do not depend on them.
# --------------------------------------------------------------------------
def pin_linearity():
    rng = np.random.default_rng(9)
    c1 = rand_case(rng, T=22, dk=8, dv=6)
    c2 = dict(c1, v=rng.standard_normal(c1["v"].shape),
              initial_state=rng.standard_normal(c1["initial_state"].shape))
    a = -1.7
    c3 = dict(c1, v=a * c1["v"] + c2["v"], initial_state=a * c1["initial_state"] + c2["initial_state"])
    o1, s1 = oracle.recurrent(**c1)
    o2, s2 = oracle.recurrent(**c2)
    o3, s3 = oracle.recurrent(**c3)
    assert rel(o3, a * o1 + o2) < TOL and rel(s3, a * s1 + s2) < TOL


# --------------------------------------------------------------------------
# (ix) orthonormal keys, g = 0: the keys never interfere, so
#      S_t = S0 + sum_{s<=t} k_s delta_s^T with delta_s = beta_s (v_s - k_s^T S0).
# --------------------------------------------------------------------------
def pin_orthonormal_keys():
    rng = np.random.default_rng(10)
    dk, dv, T = 8, 5, 6
    c = rand_case(rng, T=T, dk=dk, dv=dv, gate="zero")
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    c["k"] = Qm[:, :T].T.reshape(T, 1, dk)
    out, sf = oracle.recurrent(**c, qk_l2norm=False, scale=1.0)
    S0 = c["initial_state"][0, 0]
    S = S0.copy()
    for t in range(T):
        kk = c["k"][t, 0]
        S = S + np.outer(kk, c["beta"][t, 0] * (c["v"][t, 0] - kk @ S0))
        assert rel(out[t, 0], S.T @ c["q"][t, 0]) < TOL
    assert rel(sf[0, 0], S) < TOL


# --------------------------------------------------------------------------
# (x) the Dv columns are independent: permuting the columns of v and S0
#     permutes those of the output and the final state.
# --------------------------------------------------------------------------
def pin_dv_columns_independent():
    rng = np.random.default_rng(11)
    c = rand_case(rng, T=26, dk=8, dv=7)
    perm = rng.permutation(7)
    o, s = oracle.recurrent(**c)
    cp = dict(c, v=c["v"][..., perm], initial_state=c["initial_state"][..., perm])
    op, sp = oracle.recurrent(**cp)
    assert rel(op, o[..., perm]) < TOL and rel(sp, s[..., perm]) < TOL
    cs = dict(c, v=c["v"][..., :3], initial_state=c["initial_state"][..., :3])
    os_, ss = oracle.recurrent(**cs)
    assert rel(os_, o[..., :3]) < TOL and rel(ss, s[..., :3]) < TOL


# --------------------------------------------------------------------------
# (xi) the inverse: T (I - A) = I; T = sum_{k<C} A^k (A nilpotent, Neumann);
#      U = T diag(beta) V; W = diag(exp(gcum)) (I + L0)^-1 diag(beta) K with
#      L0 = strictLower(diag(beta) K K^T) (the walkthrough's similarity step).
# --------------------------------------------------------------------------
def pin_inverse_and_similarity():
    rng = np.random.default_rng(12)
    C, dk, dv = 16, 8, 5
    kh = unit_rows(rng.standard_normal((C, dk)))
    v = rng.standard_normal((C, dv))
    g = -rng.uniform(0, 0.5, size=C)
    beta = rng.uniform(0.1, 1.0, size=C)
    r = oracle.chunk_prepare(kh, v, g, beta)
    assert rel(r["gcum"], np.cumsum(g)) < TOL
    I = np.eye(C)
    assert np.max(np.abs(r["T"] @ (I - r["A"]) - I)) < 1e-10
    assert np.all(np.triu(r["A"]) == 0.0)
    neu = sum(np.linalg.matrix_power(r["A"], p) for p in range(C))
    assert np.max(np.abs(neu - r["T"])) < 1e-10
    assert rel(r["U"], r["T"] @ (beta[:, None] * v)) < TOL
    L0 = np.tril(beta[:, None] * (kh @ kh.T), -1)
    W = np.diag(np.exp(np.cumsum(g))) @ np.linalg.inv(I + L0) @ (beta[:, None] * kh)
    assert rel(r["W"], W) < 1e-10
    gam = np.exp(np.cumsum(g)[:, None] - np.cumsum(g)[None, :]) * (np.arange(C)[:, None] >= np.arange(C)[None, :])
    assert rel(r["gamma"], gam) < TOL
    L = np.tril(beta[:, None] * gam * (kh @ kh.T), -1)
    assert rel(r["T"], np.linalg.inv(I + L)) < 1e-10


def pin_gates_closed_forms():
    """Gate parametrisation (walkthrough section 4): beta = sigmoid(b),
    g = -exp(A_log) softplus(a + dt_bias), softplus(x) = log(1 + exp(x)).

    Pinned by values the definitions fix: sigmoid(0) = 1/2 and
    sigmoid(x) + sigmoid(-x) = 1; softplus(0) = ln 2, softplus(x) - softplus(-x) = x,
    d softplus/dx = sigmoid(x), softplus(x) ~ x for large x and ~ e^x for very
    negative x; A_log and dt_bias are per v-head; g <= 0.
    """
    nv = 3
    A = np.array([3.0, 0.5, 7.0])
    A_log, db = np.log(A), np.array([1.0, -0.25, 2.0])
    # a + dt_bias = 0 and b = 0 on every head
    g, beta = oracle.gates(np.tile(-db, (2, 1)), np.zeros((2, nv)), A_log, db)
    assert np.all(beta == 0.5)
    assert np.max(np.abs(g - (-A * np.log(2.0)))) < 1e-15
    # odd part of softplus and the sigmoid symmetry, on a grid of x = a + dt_bias
    xs = np.linspace(-30.0, 30.0, 121)
    a_p = xs[:, None] - db[None, :]
    a_m = -xs[:, None] - db[None, :]
    bb = np.repeat(xs[:, None], nv, axis=1)
    gp, bp = oracle.gates(a_p, bb, A_log, db)
    gm, bm = oracle.gates(a_m, -bb, A_log, db)
    sp, sm = gp / -A, gm / -A
    assert np.max(np.abs((sp - sm) - xs[:, None])) < 1e-12
    assert np.max(np.abs(bp + bm - 1.0)) < 1e-15
    assert np.all(gp <= 0.0) and np.all(gm <= 0.0)
    # derivative of softplus is the sigmoid of the same argument
    h = 1e-5
    g1, _ = oracle.gates(a_p + h, bb, A_log, db)
    g0, _ = oracle.gates(a_p - h, bb, A_log, db)
    dsp = (g1 - g0) / (-A) / (2 * h)
    assert np.max(np.abs(dsp - bp)) < 1e-8
    # tails
    gt, _ = oracle.gates(np.array([[40.0 - db[0], -40.0 - db[1], 0.0]]), np.zeros((1, nv)), A_log, db)
    assert abs(gt[0, 0] / -A[0] - 40.0) < 1e-13
    assert abs(gt[0, 1] / -A[1] / np.exp(-40.0) - 1.0) < 1e-12


def pin_gated_rmsnorm():
    """Output epilogue (walkthrough sections 1 and 6, RMSNormGated; its RMSNorm
    code in section 3): y = o / sqrt(mean(o^2) + eps) * w * silu(z).

    Pinned by what the definitions fix, not by retyping them:
    - with eps = 0 the normalised part has unit mean square over Dv;
    - eps sits inside the root: for a constant row o = c the ratio
      y / (w silu(z)) is 1 / sqrt(1 + eps / c^2) (eps outside would give c / (|c| + eps));
    - homogeneity: y(a o, a^2 eps) = y(o, eps) for a > 0, and y is linear in w;
    - the gate is SiLU of z: silu(0) = 0; silu(x) - silu(-x) = x; and
      silu(x) / silu(-x) = -exp(x), which fixes the logistic factor (x * Phi(x)
      would give -Phi(x) / Phi(-x));
    - rows are independent: permuting rows permutes y.
    """
    rng = np.random.default_rng(21)
    R, dv = 9, 16
    o = rng.standard_normal((R, dv)) * rng.uniform(0.1, 5.0, size=(R, 1))
    z = rng.standard_normal((R, dv)) * 3.0
    w = rng.uniform(0.5, 2.0, size=dv)
    y0 = oracle.gated_rmsnorm(o, z, w, eps=0.0)
    gate = oracle.gated_rmsnorm(np.ones((R, dv)), z, w, eps=0.0) / w  # = silu(z): o = 1 has rms 1
    n = y0 / (w * gate)
    assert np.max(np.abs(np.mean(n * n, axis=1) - 1.0)) < 1e-12
    # eps placement on constant rows
    for c_, eps in ((1e-3, 1e-6), (2.0, 0.5), (-0.3, 1e-2)):
        yc = oracle.gated_rmsnorm(np.full((1, dv), c_), np.full((1, dv), 2.0), np.ones(dv), eps)
        yg = oracle.gated_rmsnorm(np.ones((1, dv)), np.full((1, dv), 2.0), np.ones(dv), 0.0)
        ratio = yc / yg
        assert np.max(np.abs(ratio - np.sign(c_) / np.sqrt(1.0 + eps / c_ ** 2))) < 1e-13
    # homogeneity and linearity in w
    a = 7.5
    y1 = oracle.gated_rmsnorm(o, z, w, eps=1e-3)
    assert rel(oracle.gated_rmsnorm(a * o, z, w, eps=a * a * 1e-3), y1) < 1e-13
    assert rel(oracle.gated_rmsnorm(o, z, 3.0 * w, eps=1e-3), 3.0 * y1) < 1e-14
    # SiLU of z
    assert np.all(oracle.gated_rmsnorm(o, np.zeros_like(z), w, 1e-3) == 0.0)
    zz = np.linspace(-20.0, 20.0, dv)[None, :].repeat(R, axis=0)
    zz[:, dv // 2] = 0.7  # keep clear of x = 0
    yp = oracle.gated_rmsnorm(o, zz, w, 1e-3)
    ym = oracle.gated_rmsnorm(o, -zz, w, 1e-3)
    base = oracle.gated_rmsnorm(o, np.ones_like(zz), w, 1e-3) / \
        oracle.gated_rmsnorm(np.ones((R, dv)), np.ones_like(zz), np.ones(dv), 0.0)  # o/rms * w
    assert rel((yp - ym) / base, zz) < 1e-12
    assert np.max(np.abs(yp / ym / -np.exp(zz) - 1.0)) < 1e-12
    perm = rng.permutation(R)
    assert np.array_equal(oracle.gated_rmsnorm(o[perm], z[perm], w, 1e-3), y1[perm])


def _conv_ref_pre(x, w, bias, window):
    """Pre-activation of one channel by numpy's full convolution of [window, x]
    with the reversed taps (a cross-correlation), cut to the sequence."""
    ks = len(w)
    ext = np.concatenate([window, x])
    full = np.convolve(ext, w[::-1])  # full[m] = sum_i w[i] ext[m - (ks-1) + i]
    return full[ks: ks + len(x)] + bias


def pin_causal_conv1d():
    """Causal depthwise conv1d + SiLU (walkthrough section 3) and its conv_state.

    Pinned by numpy's own convolution (np.convolve with reversed taps, i.e. the
    cross-correlation of torch's conv1d) for the pre-activation, and by the
    logistic identities of SiLU: y(x) - y(-x) = pre and y(x) / y(-x) = -exp(pre)
    (inputs, bias and window negated together negate pre).  The state rules:
    the new conv_state is the last ksize inputs of [window, sequence]; one run
    equals the same tokens split in two with the state carried across, and
    equals one decode step per token (torch_causal_conv1d_update); channels and
    sequences are independent.
    """
    rng = np.random.default_rng(22)
    ch, ks = 5, 4
    lens = [1, 3, 4, 9, 17]
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = rng.standard_normal((T, ch))
    w = rng.standard_normal((ch, ks))
    bias = rng.standard_normal(ch)
    st = rng.standard_normal((len(lens), ch, ks))
    for window in (None, st):
        yp, sp = oracle.causal_conv1d(x, w, bias, cu, window)
        ym, _ = oracle.causal_conv1d(-x, w, -bias, cu, None if window is None else -window)
        for n, L in enumerate(lens):
            for c in range(ch):
                win = np.zeros(ks) if window is None else window[n, c]
                pre = _conv_ref_pre(x[cu[n]:cu[n + 1], c], w[c], bias[c], win)
                seg_p, seg_m = yp[cu[n]:cu[n + 1], c], ym[cu[n]:cu[n + 1], c]
                assert np.max(np.abs((seg_p - seg_m) - pre)) < 1e-12
                ok = np.abs(pre) > 1e-3
                assert np.max(np.abs(seg_p[ok] / seg_m[ok] / -np.exp(pre[ok]) - 1.0)) < 1e-11
                ext = np.concatenate([win, x[cu[n]:cu[n + 1], c]])
                assert np.array_equal(sp[n, c], ext[-ks:])
    # split with the state carried = one run; per-token decode = one run
    x1 = rng.standard_normal((23, ch))
    y_all, s_all = oracle.causal_conv1d(x1, w, bias, None, st[:1])
    ya, sa = oracle.causal_conv1d(x1[:10], w, bias, None, st[:1])
    yb, sb = oracle.causal_conv1d(x1[10:], w, bias, None, sa)
    assert rel(np.concatenate([ya, yb]), y_all) < 1e-15 and np.array_equal(sb, s_all)
    s_dec = st[:1].copy()
    for t in range(23):
        yt, s_dec = oracle.causal_conv1d(x1[t:t + 1], w, bias, None, s_dec)
        assert rel(yt, y_all[t:t + 1]) < 1e-15
    assert np.array_equal(s_dec, s_all)
    # causality: changing a later token leaves earlier outputs unchanged
    x2 = x1.copy()
    x2[15] += 1.0
    y2, _ = oracle.causal_conv1d(x2, w, bias, None, st[:1])
    assert np.array_equal(y2[:15], y_all[:15]) and not np.array_equal(y2[15], y_all[15])


# --------------------------------------------------------------------------
# Stored golden values (tests/golden/*.txt): outputs of small cases written by
# tests/golden/make_golden.py from the oracle, so a later change of the oracle's
# arithmetic shows up as a diff.  Regression only; the pins above are the proof.
# --------------------------------------------------------------------------

ALL_PINS = [
    pin_matrix_form, pin_l2norm_eps_closed_form, pin_scale_and_norm_invariance,
    pin_chunk_equals_recurrent, pin_beta_zero, pin_delta_write_exact, pin_zero_pad_invariance,
    pin_split_carry_and_varlen, pin_gqa_repeat_interleave, pin_linearity, pin_orthonormal_keys,
    pin_dv_columns_independent, pin_inverse_and_similarity, pin_gates_closed_forms,
    pin_gated_rmsnorm, pin_causal_conv1d,
]
