"""Plain fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import this package.  The product library
(``gated_deltanet_chunk_b200``) never imports it, and this package never imports
the product library: the two share no code.

The arithmetic lives in ``gdn_oracle.c`` (built to ``liboracle.so`` with gcc,
``-O2 -fopenmp``; no fast-math, so every operation is a plain IEEE fp64 op).
This module only marshals arrays:

* :func:`recurrent` -- the definition: the token-by-token gated delta rule of
  the "手撕Qwen3-Next" walkthrough, section 5(2) (torch_recurrent_gated_delta_rule).
* :func:`chunk_form` -- the same walkthrough's chunkwise algorithm, section
  5(1) steps a-g, with a generic chunk size.  Used only to pin the two forms
  against each other.
* :func:`gates` -- the layer's gate parametrisation (same walkthrough, section
  4): beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias).
* :func:`chunk_prepare` -- the intra-chunk quantities of one chunk (gate
  cumsum, decay mask, A, T = (I - A)^-1, U, W), for the inverse and similarity
  pins.
* :func:`gated_rmsnorm` -- the output epilogue (RMSNormGated, walkthrough
  sections 1 and 6): y = o / sqrt(mean(o^2) + eps) * w * silu(z).
* :func:`causal_conv1d` -- the causal depthwise conv1d + SiLU of the packed
  q|k|v channels with its conv_state window (walkthrough section 3; prefill and
  torch_causal_conv1d_update).

Inputs may be numpy arrays or CPU torch tensors of any float dtype (bf16
included); they are upcast exactly to fp64.  Outputs are fp64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# tests/test_oracle_mutants.py points this at deliberately broken builds
_LIB_OVERRIDE = os.environ.get("GDN_ORACLE_LIB_OVERRIDE")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle.so`` (gcc, fp64, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        lib.oracle_recurrent.argtypes = [i, ip, i, i, i, i, dp, dp, dp, dp, dp, dp, i,
                                         ctypes.c_double, dp, dp]
        lib.oracle_recurrent.restype = i
        lib.oracle_chunk_form.argtypes = [i, ip, i, i, i, i, i, dp, dp, dp, dp, dp, dp, i,
                                          ctypes.c_double, dp, dp]
        lib.oracle_chunk_form.restype = i
        lib.oracle_chunk_prepare.argtypes = [i, i, i, dp, dp, dp, dp, dp, dp, dp, dp, dp, dp]
        lib.oracle_gates.argtypes = [ctypes.c_int64, i, dp, dp, dp, dp, dp, dp]
        lib.oracle_chunk_prepare.restype = i
        lib.oracle_gated_rmsnorm.argtypes = [ctypes.c_int64, i, dp, dp, dp, ctypes.c_double, dp]
        lib.oracle_gated_rmsnorm.restype = i
        lib.oracle_causal_conv1d.argtypes = [i, ip, i, i, dp, dp, dp, dp, dp, dp]
        lib.oracle_causal_conv1d.restype = i
        _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU); bf16 -> fp32 -> fp64 is exact
        import torch
        x = x.detach().to("cpu")
        if x.dtype in (torch.bfloat16, torch.float16):
            x = x.float()
        x = x.double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a):
    if a is None:
        return None
    if a.dtype == np.int32:
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shapes(q, v, cu):
    T, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    if cu is None:
        cu = np.array([0, T], dtype=np.int32)
    cu = _i32(cu)
    return T, nqk, dk, nv, dv, cu


def recurrent(q, k, v, g, beta, initial_state=None, cu_seqlens=None,
              qk_l2norm=True, scale=0.0):
    """Token-loop definition.  Returns ``(out [T,Nv,Dv], final_state [N,Nv,Dk,Dv])``."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    s0 = _f64(initial_state)
    T, nqk, dk, nv, dv, cu = _shapes(q, v, cu_seqlens)
    n = len(cu) - 1
    out = np.zeros((T, nv, dv))
    sf = np.zeros((n, nv, dk, dv))
    rc = _load().oracle_recurrent(n, _ptr(cu), nqk, nv, dk, dv, _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(g), _ptr(beta), _ptr(s0), int(bool(qk_l2norm)),
                                  float(scale), _ptr(out), _ptr(sf))
    if rc:
        raise ValueError("oracle_recurrent: bad arguments (code %d)" % rc)
    return out, sf


def chunk_form(q, k, v, g, beta, chunk_size, initial_state=None, cu_seqlens=None,
               qk_l2norm=True, scale=0.0):
    """Chunkwise algorithm with chunk size ``chunk_size``.  Same outputs as :func:`recurrent`."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    s0 = _f64(initial_state)
    T, nqk, dk, nv, dv, cu = _shapes(q, v, cu_seqlens)
    n = len(cu) - 1
    out = np.zeros((T, nv, dv))
    sf = np.zeros((n, nv, dk, dv))
    rc = _load().oracle_chunk_form(n, _ptr(cu), nqk, nv, dk, dv, int(chunk_size), _ptr(q),
                                   _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
                                   int(bool(qk_l2norm)), float(scale), _ptr(out), _ptr(sf))
    if rc:
        raise ValueError("oracle_chunk_form: bad arguments (code %d)" % rc)
    return out, sf


def chunk_prepare(kh, v, g, beta):
    """Intra-chunk quantities of one chunk of already-normalised keys ``kh [C,Dk]``.

    Returns a dict with ``gcum [C]``, ``gamma [C,C]``, ``A [C,C]``, ``T [C,C]``,
    ``U [C,Dv]`` and ``W [C,Dk]``.
    """
    kh, v, g, beta = (_f64(x) for x in (kh, v, g, beta))
    C, dk = kh.shape
    dv = v.shape[1]
    res = {"gcum": np.zeros(C), "gamma": np.zeros((C, C)), "A": np.zeros((C, C)),
           "T": np.zeros((C, C)), "U": np.zeros((C, dv)), "W": np.zeros((C, dk))}
    rc = _load().oracle_chunk_prepare(C, dk, dv, _ptr(kh), _ptr(v), _ptr(g), _ptr(beta),
                                      *(_ptr(res[x]) for x in ("gcum", "gamma", "A", "T", "U", "W")))
    if rc:
        raise ValueError("oracle_chunk_prepare: bad arguments (code %d)" % rc)
    return res


def num_threads() -> int:
    """Threads the OpenMP oracle uses (OMP_NUM_THREADS, else the CPU affinity set)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env and env.isdigit():
        return int(env)
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def gates(a, b, A_log, dt_bias):
    """beta = sigmoid(b), g = -exp(A_log) softplus(a + dt_bias) in fp64 (oracle_gates).

    ``a``, ``b`` are [..., Nv]; ``A_log``, ``dt_bias`` are [Nv].  Returns (g, beta)
    as float64 numpy arrays of the shape of ``a``.
    """
    a64, b64 = _f64(a), _f64(b)
    al, db = _f64(A_log).reshape(-1), _f64(dt_bias).reshape(-1)
    nv = al.shape[0]
    if a64.shape != b64.shape or a64.shape[-1] != nv or db.shape[0] != nv:
        raise ValueError("gates: a, b [..., Nv] and A_log, dt_bias [Nv] expected")
    T = a64.size // nv
    g = np.empty_like(a64)
    beta = np.empty_like(a64)
    rc = _load().oracle_gates(T, nv, _ptr(a64), _ptr(b64), _ptr(al), _ptr(db), _ptr(g), _ptr(beta))
    if rc != 0:
        raise ValueError("oracle_gates failed (%d)" % rc)
    return g, beta


def gated_rmsnorm(o, z, weight, eps=1e-6):
    """y = o / sqrt(mean(o^2) + eps) * weight * silu(z) over the last axis (oracle_gated_rmsnorm).

    ``o`` and ``z`` have the same shape [..., Dv]; ``weight`` is [Dv].  Returns a
    float64 numpy array of that shape.
    """
    o64, z64, w64 = _f64(o), _f64(z), _f64(weight).reshape(-1)
    dv = o64.shape[-1]
    if z64.shape != o64.shape or w64.shape[0] != dv:
        raise ValueError("gated_rmsnorm: o, z [..., Dv] and weight [Dv] expected")
    y = np.empty_like(o64)
    rc = _load().oracle_gated_rmsnorm(o64.size // dv, dv, _ptr(o64), _ptr(z64), _ptr(w64),
                                      float(eps), _ptr(y))
    if rc != 0:
        raise ValueError("oracle_gated_rmsnorm: bad arguments (%d)" % rc)
    return y


def causal_conv1d(x, weight, bias=None, cu_seqlens=None, conv_state=None):
    """Causal depthwise conv1d + SiLU per sequence (oracle_causal_conv1d).

    ``x`` is [T, channels] (token-major), ``weight`` [channels, ksize], ``bias``
    [channels] or None, ``conv_state`` [N, channels, ksize] or None (zeros): the
    ksize inputs before each sequence.  Returns ``(y [T, channels],
    new_conv_state [N, channels, ksize])`` as float64 numpy arrays.
    """
    x64, w64 = _f64(x), _f64(weight)
    T, ch = x64.shape
    ks = w64.shape[1]
    if w64.shape[0] != ch:
        raise ValueError("causal_conv1d: weight [channels, ksize] expected")
    cu = _i32(np.array([0, T]) if cu_seqlens is None else cu_seqlens)
    n = len(cu) - 1
    b64 = _f64(bias)
    s64 = _f64(conv_state)
    y = np.empty_like(x64)
    s_out = np.zeros((n, ch, ks))
    rc = _load().oracle_causal_conv1d(n, _ptr(cu), ch, ks, _ptr(x64), _ptr(w64), _ptr(b64),
                                      _ptr(s64), _ptr(y), _ptr(s_out))
    if rc != 0:
        raise ValueError("oracle_causal_conv1d: bad arguments (%d)" % rc)
    return y, s_out
