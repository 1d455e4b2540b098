"""Gated delta rule (Gated DeltaNet core) on B200: thin Python binding of libgdn.so.

Every step of the computation runs in the CUDA kernels of ``libgdn.so``; this
module only marshals torch CUDA tensors into the C ABI of ``include/gdn.h``
(pointers, sizes, the current stream) and allocates outputs when the caller
does not pass them.  There is no CPU or PyTorch fallback: if the library is
missing the import fails, and if a call is rejected it raises ``GdnError``.

Functions
---------
chunk_fwd(q, k, v, g, beta, ...)       -> (out, final_state)   prefill, gdn_chunk_fwd
recurrent_step(q, k, v, g, beta, state, ...) -> out            decode, gdn_recurrent_step
chunk_fwd_gated / recurrent_step_gated                         the gate formed in-kernel
chunk_fwd_slots / recurrent_step_slots                         states in a slot-indexed pool
chunk_fwd_ex / recurrent_step_ex                               any of those fusions plus the
                                                               gated RMSNorm epilogue (gdn_ext_t)
gated_rmsnorm(o, z, weight, eps)       -> y                    the epilogue alone, gdn_gated_rmsnorm
qkv_conv_fwd / qkv_conv_update         -> (q, k, v[, state])  causal conv1d + SiLU producing q, k, v
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK = 0
STATUS_NAMES = {0: "GDN_OK", -1: "GDN_ERR_NULL", -2: "GDN_ERR_SHAPE", -3: "GDN_ERR_ALIGN",
                -4: "GDN_ERR_ALIAS", -5: "GDN_ERR_CUDA", -6: "GDN_ERR_DEVICE",
                -7: "GDN_ERR_DEVICE_TIMEOUT", -8: "GDN_ERR_SEQLENS", -9: "GDN_ERR_GATE"}
KERNELS = {"auto": 0, "simt": 1, "tc": 2}
DTYPE_F32, DTYPE_BF16 = 0, 1


class GdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s" % (what, lib().gdn_status_string(status).decode()))


class GdnParams(ctypes.Structure):
    _fields_ = [("num_qk_heads", ctypes.c_int32), ("num_v_heads", ctypes.c_int32),
                ("head_k_dim", ctypes.c_int32), ("head_v_dim", ctypes.c_int32),
                ("io_dtype", ctypes.c_int32), ("qk_l2norm", ctypes.c_int32),
                ("scale", ctypes.c_float), ("kernel", ctypes.c_int32)]


class GdnExt(ctypes.Structure):
    _fields_ = [("A_log", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p), ("slot_ids", ctypes.c_void_p),
                ("num_slots", ctypes.c_int32), ("norm_z", ctypes.c_void_p), ("norm_weight", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float), ("conv_x", ctypes.c_void_p), ("conv_state", ctypes.c_void_p),
                ("conv_weight", ctypes.c_void_p), ("conv_bias", ctypes.c_void_p),
                ("conv_kernel_size", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libgdn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                "libgdn.so is not built (expected at %s); run "
                "`python -m gated_deltanet_chunk_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
        L.gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, ip, ctypes.c_int32, ctypes.c_int64,
                                    ctypes.c_int32, vp, fp, ctypes.POINTER(GdnParams), vp]
        L.gdn_chunk_fwd.restype = ctypes.c_int
        L.gdn_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, ctypes.c_int32,
                                         ctypes.POINTER(GdnParams), vp]
        L.gdn_recurrent_step.restype = ctypes.c_int
        L.gdn_chunk_fwd_gated.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, ip, ctypes.c_int32,
                                          ctypes.c_int64, ctypes.c_int32, vp, fp,
                                          ctypes.POINTER(GdnParams), vp]
        L.gdn_chunk_fwd_gated.restype = ctypes.c_int
        L.gdn_recurrent_step_gated.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, vp, ctypes.c_int32,
                                               ctypes.POINTER(GdnParams), vp]
        L.gdn_recurrent_step_gated.restype = ctypes.c_int
        L.gdn_chunk_fwd_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, ctypes.c_int32, ip, ctypes.c_int32,
                                          ctypes.c_int64, ctypes.c_int32, vp, ctypes.POINTER(GdnParams), vp]
        L.gdn_chunk_fwd_slots.restype = ctypes.c_int
        L.gdn_recurrent_step_slots.argtypes = [vp, vp, vp, fp, fp, fp, ip, ctypes.c_int32, vp, ctypes.c_int32,
                                               ctypes.POINTER(GdnParams), vp]
        L.gdn_recurrent_step_slots.restype = ctypes.c_int
        L.gdn_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, ip, ctypes.c_int32, ctypes.c_int64,
                                       ctypes.c_int32, vp, fp, ctypes.POINTER(GdnParams),
                                       ctypes.POINTER(GdnExt), vp]
        L.gdn_chunk_fwd_ex.restype = ctypes.c_int
        L.gdn_recurrent_step_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, ctypes.c_int32,
                                            ctypes.POINTER(GdnParams), ctypes.POINTER(GdnExt), vp]
        L.gdn_recurrent_step_ex.restype = ctypes.c_int
        L.gdn_gated_rmsnorm.argtypes = [vp, vp, fp, ctypes.c_float, vp, ctypes.c_int64, ctypes.c_int32,
                                        ctypes.c_int32, vp]
        L.gdn_gated_rmsnorm.restype = ctypes.c_int
        L.gdn_qkv_conv_fwd.argtypes = [vp, fp, fp, vp, ip, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32,
                                       vp, vp, vp, vp, ctypes.POINTER(GdnParams), vp]
        L.gdn_qkv_conv_fwd.restype = ctypes.c_int
        L.gdn_qkv_conv_update.argtypes = [vp, fp, fp, vp, ip, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          vp, vp, vp, ctypes.POINTER(GdnParams), vp]
        L.gdn_qkv_conv_update.restype = ctypes.c_int
        L.gdn_selftest_wait_timeout.argtypes = [ctypes.c_int64, vp]
        L.gdn_selftest_wait_timeout.restype = ctypes.c_int
        L.gdn_device_status.argtypes = [vp]
        L.gdn_device_status.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_version.argtypes = []
        L.gdn_version.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_params(nqk, nv, dk, dv, io_bf16, qk_l2norm=True, scale=0.0, kernel="auto") -> GdnParams:
    return GdnParams(int(nqk), int(nv), int(dk), int(dv), DTYPE_BF16 if io_bf16 else DTYPE_F32,
                     1 if qk_l2norm else 0, float(scale), KERNELS[kernel])


def _chunk_call(name, gate, q, k, v, initial_state, cu_seqlens, chunk_size, out, final_state,
                output_final_state, num_seqs, qk_l2norm, scale, kernel, stream, check):
    import torch
    T, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (num_seqs or 1)
    if out is None:
        out = torch.empty((T, nv, dv), dtype=v.dtype, device=v.device)
    if final_state is None and output_final_state:
        final_state = torch.empty((n, nv, dk, dv), dtype=torch.float32, device=v.device)
    p = make_params(nqk, nv, dk, dv, q.dtype == torch.bfloat16, qk_l2norm, scale, kernel)
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in gate], _ptr(initial_state),
                              _ptr(cu_seqlens), int(n), int(T), int(chunk_size), _ptr(out),
                              _ptr(final_state), ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, name)
    return out, final_state


def chunk_fwd(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk_size=64,
              out=None, final_state=None, output_final_state=True, num_seqs=None,
              qk_l2norm=True, scale=0.0, kernel="auto", stream=None, check=True):
    """Chunked gated delta rule over a packed batch (``gdn_chunk_fwd``).

    q, k [T, Nqk, Dk] and v [T, Nv, Dv] (bf16 or fp32, CUDA, contiguous);
    g, beta [T, Nv] fp32; initial_state [N, Nv, Dk, Dv] fp32 or None;
    cu_seqlens [N+1] int32 or None (then ``num_seqs`` equal sequences, default 1).
    Returns ``(out, final_state)``; final_state is None when not requested.
    """
    return _chunk_call("gdn_chunk_fwd", (g, beta), q, k, v, initial_state, cu_seqlens, chunk_size,
                       out, final_state, output_final_state, num_seqs, qk_l2norm, scale, kernel,
                       stream, check)


def chunk_fwd_gated(q, k, v, a, b, A_log, dt_bias, initial_state=None, cu_seqlens=None,
                    chunk_size=64, out=None, final_state=None, output_final_state=True,
                    num_seqs=None, qk_l2norm=True, scale=0.0, kernel="auto", stream=None,
                    check=True):
    """``chunk_fwd`` with the gate formed in-kernel (``gdn_chunk_fwd_gated``).

    a, b [T, Nv] fp32 raw projections; A_log, dt_bias [Nv] fp32:
    beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias).
    """
    return _chunk_call("gdn_chunk_fwd_gated", (a, b, A_log, dt_bias), q, k, v, initial_state,
                       cu_seqlens, chunk_size, out, final_state, output_final_state, num_seqs,
                       qk_l2norm, scale, kernel, stream, check)


def _step_call(name, gate, q, k, v, state, out, qk_l2norm, scale, stream, check):
    import torch
    N, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    if out is None:
        out = torch.empty((N, nv, dv), dtype=v.dtype, device=v.device)
    p = make_params(nqk, nv, dk, dv, q.dtype == torch.bfloat16, qk_l2norm, scale)
    rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), *[_ptr(x) for x in gate], _ptr(state),
                              _ptr(out), int(N), ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, name)
    return out


def recurrent_step(q, k, v, g, beta, state, out=None, qk_l2norm=True, scale=0.0, stream=None,
                   check=True):
    """One decode token per sequence (``gdn_recurrent_step``); ``state`` is updated in place.

    q, k [N, Nqk, Dk], v [N, Nv, Dv], g, beta [N, Nv], state [N, Nv, Dk, Dv] fp32.
    Returns out [N, Nv, Dv].
    """
    return _step_call("gdn_recurrent_step", (g, beta), q, k, v, state, out, qk_l2norm, scale,
                      stream, check)


def recurrent_step_gated(q, k, v, a, b, A_log, dt_bias, state, out=None, qk_l2norm=True,
                         scale=0.0, stream=None, check=True):
    """``recurrent_step`` with the gate formed in-kernel (``gdn_recurrent_step_gated``).

    a, b [N, Nv] fp32 raw projections; A_log, dt_bias [Nv] fp32.
    """
    return _step_call("gdn_recurrent_step_gated", (a, b, A_log, dt_bias), q, k, v, state, out,
                      qk_l2norm, scale, stream, check)


def selftest_wait_timeout(limit_us=2000, stream=None) -> int:
    """Launch the failure-detection self-test (``gdn_selftest_wait_timeout``); then
    ``device_status()`` reports GDN_ERR_DEVICE_TIMEOUT once."""
    return lib().gdn_selftest_wait_timeout(int(limit_us), _stream(stream))


def device_status(stream=None) -> int:
    """Synchronise the stream and return the library's device status (``gdn_device_status``)."""
    return lib().gdn_device_status(_stream(stream))


def chunk_fwd_slots(q, k, v, g, beta, state_pool, slot_ids, cu_seqlens=None, chunk_size=64, out=None,
                    num_seqs=None, qk_l2norm=True, scale=0.0, kernel="auto", stream=None, check=True):
    """Chunked forward with the states in a slot-indexed pool, updated in place (``gdn_chunk_fwd_slots``).

    state_pool [P, Nv, Dk, Dv] fp32; slot_ids [N] int32 (ids outside [0, P) mark padding
    sequences); cu_seqlens [N+1] or None.  Returns out [T, Nv, Dv].
    """
    import torch
    T, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    n = slot_ids.numel()
    if out is None:
        out = torch.empty((T, nv, dv), dtype=v.dtype, device=v.device)
    p = make_params(nqk, nv, dk, dv, q.dtype == torch.bfloat16, qk_l2norm, scale, kernel)
    rc = lib().gdn_chunk_fwd_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                   _ptr(slot_ids), int(state_pool.shape[0]), _ptr(cu_seqlens), int(n),
                                   int(T), int(chunk_size), _ptr(out), ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_fwd_slots")
    return out


def recurrent_step_slots(q, k, v, g, beta, state_pool, slot_ids, out=None, qk_l2norm=True, scale=0.0,
                         stream=None, check=True):
    """One decode token per sequence with slot-indexed states (``gdn_recurrent_step_slots``)."""
    import torch
    N, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    if out is None:
        out = torch.empty((N, nv, dv), dtype=v.dtype, device=v.device)
    p = make_params(nqk, nv, dk, dv, q.dtype == torch.bfloat16, qk_l2norm, scale)
    rc = lib().gdn_recurrent_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_pool),
                                        _ptr(slot_ids), int(state_pool.shape[0]), _ptr(out), int(N),
                                        ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrent_step_slots")
    return out


def make_ext(A_log=None, dt_bias=None, slot_ids=None, num_slots=0, norm_z=None, norm_weight=None,
             norm_eps=1e-6, conv_x=None, conv_state=None, conv_weight=None, conv_bias=None) -> GdnExt:
    """The gdn_ext_t block: fused gate, slot pool, gated RMSNorm epilogue, fused conv (each optional)."""
    p = lambda t: None if t is None else t.data_ptr()
    return GdnExt(p(A_log), p(dt_bias), p(slot_ids), int(num_slots), p(norm_z), p(norm_weight),
                  float(norm_eps), p(conv_x), p(conv_state), p(conv_weight), p(conv_bias),
                  int(conv_weight.shape[1]) if conv_weight is not None else 0)


def chunk_fwd_ex(q, k, v, g, beta, initial_state=None, cu_seqlens=None, chunk_size=64, out=None,
                 final_state=None, output_final_state=True, num_seqs=None, qk_l2norm=True, scale=0.0,
                 kernel="auto", A_log=None, dt_bias=None, slot_ids=None, norm_z=None, norm_weight=None,
                 norm_eps=1e-6, stream=None, check=True):
    """``chunk_fwd`` with any of the fusions of ``gdn_chunk_fwd_ex``.

    A_log, dt_bias: the g, beta arguments are the raw projections a, b.
    slot_ids: ``initial_state`` is a state pool [P, Nv, Dk, Dv], updated in place.
    norm_z [T, Nv, Dv] (dtype of v), norm_weight [Dv] fp32: out holds
    o / sqrt(mean(o^2) + norm_eps) * norm_weight * silu(norm_z) per row.
    Returns ``(out, final_state)``.
    """
    import torch
    T, nqk, dk = q.shape
    nv, dv = v.shape[1], v.shape[2]
    if slot_ids is not None:
        n = slot_ids.numel()
        final_state = initial_state
    else:
        n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (num_seqs or 1)
        if final_state is None and output_final_state:
            final_state = torch.empty((n, nv, dk, dv), dtype=torch.float32, device=v.device)
    if out is None:
        out = torch.empty((T, nv, dv), dtype=v.dtype, device=v.device)
    p = make_params(nqk, nv, dk, dv, q.dtype == torch.bfloat16, qk_l2norm, scale, kernel)
    x = make_ext(A_log, dt_bias, slot_ids, 0 if initial_state is None or slot_ids is None
                 else initial_state.shape[0], norm_z, norm_weight, norm_eps)
    rc = lib().gdn_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                                _ptr(cu_seqlens), int(n), int(T), int(chunk_size), _ptr(out),
                                _ptr(final_state), ctypes.byref(p), ctypes.byref(x), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_chunk_fwd_ex")
    return out, final_state


def recurrent_step_ex(q, k, v, g, beta, state, out=None, qk_l2norm=True, scale=0.0, A_log=None,
                      dt_bias=None, slot_ids=None, norm_z=None, norm_weight=None, norm_eps=1e-6,
                      conv_x=None, conv_state=None, conv_weight=None, conv_bias=None, shapes=None,
                      stream=None, check=True):
    """``recurrent_step`` with any of the fusions of ``gdn_recurrent_step_ex`` (see chunk_fwd_ex).

    With the conv fused, pass q = k = v = None, ``conv_x`` [N, C], ``conv_state``
    [N or P, C, K] (updated in place), ``conv_weight`` [C, K], ``conv_bias`` and
    ``shapes=(nqk, nv, dk, dv)``.
    """
    import torch
    if conv_x is not None:
        nqk, nv, dk, dv = shapes
        N = conv_x.shape[0]
        io_bf16, dev = conv_x.dtype == torch.bfloat16, conv_x.device
    else:
        N, nqk, dk = q.shape
        nv, dv = v.shape[1], v.shape[2]
        io_bf16, dev = q.dtype == torch.bfloat16, v.device
    if out is None:
        out = torch.empty((N, nv, dv), dtype=torch.bfloat16 if io_bf16 else torch.float32, device=dev)
    p = make_params(nqk, nv, dk, dv, io_bf16, qk_l2norm, scale)
    x = make_ext(A_log, dt_bias, slot_ids, state.shape[0] if slot_ids is not None else 0, norm_z,
                 norm_weight, norm_eps, conv_x, conv_state, conv_weight, conv_bias)
    rc = lib().gdn_recurrent_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), _ptr(out),
                                     int(N), ctypes.byref(p), ctypes.byref(x), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrent_step_ex")
    return out


def gated_rmsnorm(o, z, weight, eps=1e-6, out=None, stream=None, check=True):
    """y = o / sqrt(mean(o^2) + eps) * weight * silu(z) over the last axis (``gdn_gated_rmsnorm``).

    o, z [..., D] (bf16 or fp32, same dtype, CUDA, contiguous; D in {64, 128});
    weight [D] fp32.  ``out`` may be ``o`` (in place).
    """
    import torch
    dim = o.shape[-1]
    if out is None:
        out = torch.empty_like(o)
    rc = lib().gdn_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(weight), float(eps), _ptr(out), int(o.numel() // dim),
                                 int(dim), DTYPE_BF16 if o.dtype == torch.bfloat16 else DTYPE_F32,
                                 _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_gated_rmsnorm")
    return out


def _qkv_out(rows, nqk, nv, dk, dv, dtype, device):
    import torch
    return (torch.empty((rows, nqk, dk), dtype=dtype, device=device),
            torch.empty((rows, nqk, dk), dtype=dtype, device=device),
            torch.empty((rows, nv, dv), dtype=dtype, device=device))


def qkv_conv_fwd(mixed_qkv, weight, nqk, nv, dk, dv, bias=None, conv_state=None, cu_seqlens=None,
                 num_seqs=None, output_state=True, state_out=None, stream=None, check=True):
    """Causal depthwise conv1d + SiLU of packed [q | k | v] channels (``gdn_qkv_conv_fwd``).

    mixed_qkv [T, C] (bf16 or fp32), weight [C, K] fp32, bias [C] fp32 or None,
    conv_state [N, C, K] or None (zeros).  Returns ``(q, k, v, state)`` with q, k
    [T, Nqk, Dk], v [T, Nv, Dv] and the new conv_state [N, C, K] (None unless
    requested; ``state_out=conv_state`` updates it in place).
    """
    import torch
    T, C = mixed_qkv.shape
    K = weight.shape[1]
    n = (cu_seqlens.numel() - 1) if cu_seqlens is not None else (num_seqs or 1)
    q, k, v = _qkv_out(T, nqk, nv, dk, dv, mixed_qkv.dtype, mixed_qkv.device)
    if state_out is None and output_state:
        state_out = torch.empty((n, C, K), dtype=mixed_qkv.dtype, device=mixed_qkv.device)
    p = make_params(nqk, nv, dk, dv, mixed_qkv.dtype == torch.bfloat16)
    rc = lib().gdn_qkv_conv_fwd(_ptr(mixed_qkv), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(cu_seqlens),
                                int(n), int(T), int(K), _ptr(q), _ptr(k), _ptr(v), _ptr(state_out),
                                ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_qkv_conv_fwd")
    return q, k, v, state_out


def qkv_conv_update(mixed_qkv, weight, conv_state, nqk, nv, dk, dv, bias=None, slot_ids=None, out=None,
                    stream=None, check=True):
    """One decode token per sequence through the conv (``gdn_qkv_conv_update``); conv_state in place.

    mixed_qkv [N, C]; conv_state [N, C, K] (or a pool [P, C, K] with slot_ids [N] int32).
    Returns ``(q, k, v)`` with q, k [N, Nqk, Dk] and v [N, Nv, Dv].
    """
    import torch
    N, C = mixed_qkv.shape
    K = weight.shape[1]
    q, k, v = out if out is not None else _qkv_out(N, nqk, nv, dk, dv, mixed_qkv.dtype, mixed_qkv.device)
    p = make_params(nqk, nv, dk, dv, mixed_qkv.dtype == torch.bfloat16)
    rc = lib().gdn_qkv_conv_update(_ptr(mixed_qkv), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(slot_ids),
                                   int(conv_state.shape[0]) if slot_ids is not None else 0, int(N), int(K),
                                   _ptr(q), _ptr(k), _ptr(v), ctypes.byref(p), _stream(stream))
    if check and rc != GDN_OK:
        raise GdnError(rc, "gdn_qkv_conv_update")
    return q, k, v
