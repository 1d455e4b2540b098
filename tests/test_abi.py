"""The C-ABI library: it loads, exports every symbol include/gdn.h declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


@pytest.fixture(scope="module")
def L():
    from gated_deltanet_chunk_b200 import build
    build.build()
    import gated_deltanet_chunk_b200 as g
    return g.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", src)))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("gdn_chunk_fwd", "gdn_recurrent_step", "gdn_status_string", "gdn_device_status",
              "gdn_version"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_header_is_plain_c_and_links(L, tmp_path):
    """include/gdn.h is a C header (no torch or C++ types): a C99 file that calls every declared
    entry point compiles with -Wall -Werror and links against libgdn.so with no undefined symbol."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = tmp_path / "use_all.c"
    src.write_text('#include "gdn.h"\n'
                   "typedef void (*fn)(void);\n"
                   "fn table[] = {" + ", ".join("(fn)%s" % n for n in names) + "};\n")
    obj, lib = tmp_path / "use_all.o", tmp_path / "libuse.so"
    cc = ["gcc", "-std=c99", "-Wall", "-Werror", "-fPIC", "-I", os.path.join(ROOT, "include"), "-c", str(src),
          "-o", str(obj)]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    libdir = os.path.join(ROOT, "gated_deltanet_chunk_b200")
    ld = ["gcc", "-shared", "-o", str(lib), str(obj), "-L", libdir, "-lgdn", "-Wl,--no-undefined",
          "-Wl,-rpath," + libdir]
    r = subprocess.run(ld, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_version_and_status_strings(L):
    assert L.gdn_version() >> 16 == 1
    for code in range(-9, 1):
        s = L.gdn_status_string(code).decode()
        assert s.startswith("GDN") and "unknown" not in s
    assert "SEQLENS" in L.gdn_status_string(-8).decode() and "GATE" in L.gdn_status_string(-9).decode()
    assert "unknown" in L.gdn_status_string(5).decode()


# Fake, never-dereferenced, 16-byte aligned addresses: validation must reject
# these calls on the host before it touches the device or the memory.
A = 0x100000


def _p(**kw):
    import gated_deltanet_chunk_b200 as g
    base = dict(nqk=2, nv=4, dk=128, dv=128, io_bf16=True)
    base.update(kw)
    return g.make_params(base["nqk"], base["nv"], base["dk"], base["dv"], base["io_bf16"])


def _chunk(L, p, q=A, k=A + 0x1000000, v=A + 0x2000000, g=A + 0x3000000, b=A + 0x4000000,
           s0=None, cu=None, n=2, T=256, C=64, out=A + 0x5000000, sf=None):
    vp = ctypes.c_void_p
    return L.gdn_chunk_fwd(vp(q), vp(k), vp(v), vp(g), vp(b), vp(s0), vp(cu), n, T, C, vp(out),
                           vp(sf), ctypes.byref(p) if p is not None else None, None)


def test_validation_rejects_before_launch(L):
    # NULL params / pointers
    assert _chunk(L, None) == -1
    assert _chunk(L, _p(), q=None) == -1
    assert _chunk(L, _p(), out=None) == -1
    # shapes
    assert _chunk(L, _p(nqk=3, nv=4)) == -2            # Nv % Nqk != 0
    assert _chunk(L, _p(dk=96)) == -2                  # head dim
    assert _chunk(L, _p(dv=32)) == -2
    assert _chunk(L, _p(), C=32) == -2                 # chunk size
    assert _chunk(L, _p(), n=0) == -2                  # no sequences
    assert _chunk(L, _p(), T=255, n=2) == -2           # uneven split without cu_seqlens
    assert _chunk(L, _p(), T=-1) == -2
    # alignment
    assert _chunk(L, _p(), q=A + 4) == -3
    assert _chunk(L, _p(), cu=A + 0x6000008) == -3
    # aliasing: out over v; final_state over q; final_state partially over initial_state
    assert _chunk(L, _p(), out=A + 0x2000000) == -4
    assert _chunk(L, _p(), sf=A) == -4
    assert _chunk(L, _p(), s0=A + 0x7000000, sf=A + 0x7000000 + 4096) == -4


def test_recurrent_validation(L):
    vp = ctypes.c_void_p
    p = _p()
    assert L.gdn_recurrent_step(vp(A), vp(A), vp(A), vp(A), vp(A), None, vp(A), 4, ctypes.byref(p), None) == -1
    assert L.gdn_recurrent_step(vp(A), vp(A + 0x100000), vp(A + 0x200000), vp(A + 0x300000), vp(A + 0x400000),
                                vp(A + 0x500000), vp(A + 0x500000), 4, ctypes.byref(p), None) == -4
    assert L.gdn_recurrent_step(vp(A), vp(A + 0x100000), vp(A + 0x200000), vp(A + 0x300000), vp(A + 0x400000),
                                vp(A + 0x500000), vp(A + 0x900002), 4, ctypes.byref(p), None) == -3
    bad = _p(nqk=5, nv=4)
    assert L.gdn_recurrent_step(vp(A), vp(A), vp(A), vp(A), vp(A), vp(A), vp(A), 4, ctypes.byref(bad), None) == -2


def test_valid_call_without_gpu_launches_nothing(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("only meaningful without a GPU (the fake pointers must never reach a kernel)")
    rc = _chunk(L, _p())
    assert rc in (-5, -6)  # the device check fails: no kernel is launched


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import gated_deltanet_chunk_b200 as g
    monkeypatch.setattr(g, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(g, "_lib", None)
    with pytest.raises(ImportError):
        g.lib()


def _chunk_gated(L, p, al=A + 0x8000000, db=A + 0x8001000, out=A + 0x5000000):
    vp = ctypes.c_void_p
    return L.gdn_chunk_fwd_gated(vp(A), vp(A + 0x1000000), vp(A + 0x2000000), vp(A + 0x3000000),
                                 vp(A + 0x4000000), vp(al), vp(db), None, None, 2, 256, 64, vp(out),
                                 None, ctypes.byref(p), None)


def test_gated_validation(L):
    p = _p()
    assert _chunk_gated(L, p, al=None) == -1            # A_log and dt_bias are required
    assert _chunk_gated(L, p, db=None) == -1
    assert _chunk_gated(L, p, al=A + 0x8000002) == -3   # 4-byte alignment
    assert _chunk_gated(L, p, out=A + 0x8000000) == -4  # out over A_log
    vp = ctypes.c_void_p
    assert L.gdn_recurrent_step_gated(vp(A), vp(A + 0x100000), vp(A + 0x200000), vp(A + 0x300000),
                                      vp(A + 0x400000), None, vp(A + 0x500000), vp(A + 0x600000),
                                      vp(A + 0x900000), 4, ctypes.byref(p), None) == -1
    import torch
    if not torch.cuda.is_available():
        assert _chunk_gated(L, p) in (-5, -6)          # valid: stops at the device check


def test_slots_validation(L):
    vp, p = ctypes.c_void_p, _p()

    def chunk(pool=A + 0x8000000, slots=A + 0x9000000, nslots=16, out=A + 0x5000000):
        return L.gdn_chunk_fwd_slots(vp(A), vp(A + 0x1000000), vp(A + 0x2000000), vp(A + 0x3000000),
                                     vp(A + 0x4000000), vp(pool), vp(slots), nslots, None, 2, 256, 64,
                                     vp(out), ctypes.byref(p), None)
    assert chunk(pool=None) == -1
    assert chunk(slots=None) == -1
    assert chunk(nslots=0) == -2
    assert chunk(slots=A + 0x9000002) == -3          # 4-byte alignment of the slot ids
    assert chunk(out=A + 0x8000000) == -4            # out over the pool
    assert L.gdn_recurrent_step_slots(vp(A), vp(A + 0x100000), vp(A + 0x200000), vp(A + 0x300000),
                                      vp(A + 0x400000), vp(A + 0x500000), None, 8, vp(A + 0x900000), 4,
                                      ctypes.byref(p), None) == -1
    import torch
    if not torch.cuda.is_available():
        assert chunk() in (-5, -6)                   # valid: stops at the device check


def _chunk_ex(L, p, x, s0=None, sf=None, out=A + 0x5000000):
    vp = ctypes.c_void_p
    return L.gdn_chunk_fwd_ex(vp(A), vp(A + 0x1000000), vp(A + 0x2000000), vp(A + 0x3000000),
                              vp(A + 0x4000000), vp(s0), None, 2, 256, 64, vp(out), vp(sf),
                              ctypes.byref(p), ctypes.byref(x) if x is not None else None, None)


def test_ext_validation(L):
    import gated_deltanet_chunk_b200 as g
    import torch
    p = _p()
    Z, W = A + 0xA000000, A + 0xB000000

    def ext(**kw):
        x = g.GdnExt()
        for k_, v_ in kw.items():
            setattr(x, k_, v_)
        return x
    assert _chunk_ex(L, p, ext(A_log=A + 0x8000000)) == -1                     # half a gate
    assert _chunk_ex(L, p, ext(norm_z=Z)) == -1                                # norm without weight
    assert _chunk_ex(L, p, ext(norm_z=Z, norm_weight=W, norm_eps=-1.0)) == -2   # negative eps
    assert _chunk_ex(L, p, ext(norm_z=Z, norm_weight=W, norm_eps=float("nan"))) == -2
    assert _chunk_ex(L, p, ext(norm_z=Z + 8, norm_weight=W)) == -3             # 16-byte alignment
    assert _chunk_ex(L, p, ext(norm_z=Z, norm_weight=W + 4)) == -3
    assert _chunk_ex(L, p, ext(norm_z=Z, norm_weight=W), out=Z) == -4          # out over z
    assert _chunk_ex(L, p, ext(norm_z=A + 0x5000000 + 4096, norm_weight=W)) == -4
    assert _chunk_ex(L, p, ext(slot_ids=A + 0x9000000, num_slots=0),
                     s0=A + 0x8000000, sf=A + 0x8000000) == -2                 # empty pool
    assert _chunk_ex(L, p, ext(slot_ids=A + 0x9000000, num_slots=8), s0=A + 0x8000000) == -1  # pool != final
    vp = ctypes.c_void_p
    x = ext(norm_z=Z, norm_weight=W)
    assert L.gdn_recurrent_step_ex(vp(A), vp(A + 0x100000), vp(A + 0x200000), vp(A + 0x300000),
                                   vp(A + 0x400000), vp(A + 0x500000), vp(Z), 4, ctypes.byref(p),
                                   ctypes.byref(x), None) == -4                # out over z
    if not torch.cuda.is_available():
        assert _chunk_ex(L, p, None) in (-5, -6)                              # NULL ext = plain call
        assert _chunk_ex(L, p, ext(norm_z=Z, norm_weight=W, norm_eps=1e-6)) in (-5, -6)


def test_gated_rmsnorm_validation(L):
    import torch
    vp = ctypes.c_void_p
    O, Z, W, Y = A, A + 0x1000000, A + 0x2000000, A + 0x3000000

    def call(o=O, z=Z, w=W, eps=1e-6, y=Y, rows=100, dim=128, dt=1):
        return L.gdn_gated_rmsnorm(vp(o), vp(z), vp(w), eps, vp(y), rows, dim, dt, None)
    assert call(z=None) == -1
    assert call(o=None, z=None, w=None, y=None, rows=0) == 0   # empty: nothing to do
    assert call(dim=96) == -2
    assert call(rows=-1) == -2
    assert call(dt=7) == -2
    assert call(eps=-1e-3) == -2
    assert call(o=O + 2) == -3
    assert call(y=Z) == -4                    # y over z
    assert call(y=O + 256) == -4              # y partly over o (in place needs y == o exactly)
    if not torch.cuda.is_available():
        assert call(y=O) in (-5, -6)          # in place is valid: stops at the device check
        assert call() in (-5, -6)


def test_conv_validation(L):
    import torch
    vp = ctypes.c_void_p
    p = _p(nqk=2, nv=4, dk=128, dv=128)                 # C = 1024
    X, Wt, Q, K_, V = A, A + 0x1000000, A + 0x2000000, A + 0x3000000, A + 0x4000000

    def fwd(x=X, w=Wt, b=None, si=None, cu=None, n=2, T=256, ks=4, q=Q, k=K_, v=V, so=None, pp=p):
        return L.gdn_qkv_conv_fwd(vp(x), vp(w), vp(b), vp(si), vp(cu), n, T, ks, vp(q), vp(k), vp(v), vp(so),
                                  ctypes.byref(pp), None)
    assert fwd(x=None) == -1
    assert fwd(q=None) == -1
    assert fwd(ks=0) == -2 and fwd(ks=5) == -2          # taps in [1, 4]
    assert fwd(T=255) == -2                             # uneven split without cu_seqlens
    assert fwd(pp=_p(nqk=3, nv=4)) == -2
    assert fwd(x=X + 8) == -3
    assert fwd(w=Wt + 2) == -3
    assert fwd(w=Wt + 4) == -3                          # taps are read as 16-byte vectors
    assert fwd(q=X) == -4                               # q over the input
    assert fwd(k=Q + 4096) == -4                        # k over q
    assert fwd(si=A + 0x5000000, so=A + 0x5000000 + 64) == -4   # partial state overlap
    assert fwd(so=Wt) == -4                             # state over the weight

    def upd(st=A + 0x5000000, slots=None, ns=0, q=Q):
        return L.gdn_qkv_conv_update(vp(X), vp(Wt), None, vp(st), vp(slots), ns, 4, 4, vp(q), vp(K_), vp(V),
                                     ctypes.byref(p), None)
    assert upd(st=None) == -1
    assert upd(slots=A + 0x6000000, ns=0) == -2
    assert upd(slots=A + 0x6000002, ns=8) == -3
    assert upd(q=A + 0x5000000) == -4                   # q over the state
    if not torch.cuda.is_available():
        assert fwd() in (-5, -6)
        assert fwd(si=A + 0x5000000, so=A + 0x5000000) in (-5, -6)   # in place is valid
        assert upd() in (-5, -6)


def test_ext_conv_validation(L):
    import gated_deltanet_chunk_b200 as g
    import torch
    vp = ctypes.c_void_p
    CX, CS, CW = A + 0xC000000, A + 0xD000000, A + 0xE000000

    def step(q=None, pp=None, **kw):
        x = g.GdnExt(conv_x=CX, conv_state=CS, conv_weight=CW, conv_kernel_size=4)
        for k_, v_ in kw.items():
            setattr(x, k_, v_)
        pp = pp or _p()
        return L.gdn_recurrent_step_ex(vp(q), None, None, vp(A + 0x300000), vp(A + 0x400000), vp(A + 0x500000),
                                       vp(A + 0x900000), 4, ctypes.byref(pp), ctypes.byref(x), None)
    assert step(q=A) == -2                                     # q given with the fused conv
    assert step(conv_state=None) == -1
    assert step(conv_kernel_size=5) == -2
    assert step(pp=_p(nqk=1, nv=16)) == -2                     # group of 16 v-heads: no cluster that large
    assert step(conv_x=CX + 8) == -3
    assert step(conv_state=A + 0x500000) == -4                 # conv state over the recurrent state
    assert step(conv_x=A + 0x900000) == -4                     # out over the projection
    x = g.GdnExt(conv_x=CX, conv_state=CS, conv_weight=CW, conv_kernel_size=4)
    assert L.gdn_chunk_fwd_ex(vp(A), vp(A + 0x1000000), vp(A + 0x2000000), vp(A + 0x3000000), vp(A + 0x4000000),
                              None, None, 2, 256, 64, vp(A + 0x5000000), None, ctypes.byref(_p()),
                              ctypes.byref(x), None) == -2         # no fused conv on the chunked call
    if not torch.cuda.is_available():
        assert step() in (-5, -6)


def test_selftest_wait_timeout_validation(L):
    import torch
    assert L.gdn_selftest_wait_timeout(0, None) == -2
    assert L.gdn_selftest_wait_timeout(2000001, None) == -2
    if not torch.cuda.is_available():
        assert L.gdn_selftest_wait_timeout(1000, None) in (-5, -6)


def test_empty_batch_accepts_null_token_tensors(L):
    import torch
    vp = ctypes.c_void_p
    p = _p()
    S0, SF = A + 0x7000000, A + 0x8000000
    rc = L.gdn_chunk_fwd(None, None, None, None, None, vp(S0), None, 2, 0, 64, None, vp(SF), ctypes.byref(p), None)
    rc_tokens = L.gdn_chunk_fwd(None, None, None, None, None, vp(S0), None, 2, 256, 64, None, vp(SF),
                                ctypes.byref(p), None)
    assert rc_tokens == -1                        # with tokens the tensors are required
    rc_conv = L.gdn_qkv_conv_fwd(None, vp(A), None, None, None, 2, 0, 4, None, None, None, vp(SF),
                                 ctypes.byref(p), None)
    if not torch.cuda.is_available():
        assert rc in (-5, -6) and rc_conv in (-5, -6)   # valid: stops at the device check
