"""Host-only checks of the C ABI: libgdn.so loads without a GPU, exports every
function include/gdn.h declares, and its guards refuse bad arguments with the
named error before anything is launched (no compute call is made here)."""
import ctypes
import os
import re

import pytest

from linear_attention_ssm_gdn_b200 import _lib
from linear_attention_ssm_gdn_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

# Fake, 16-byte-aligned device addresses: every call below must be refused by a
# host-side guard before it could touch them.
P = 0x10000
NULL = None


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_version_and_last_error(lib):
    assert lib.gdn_version().decode().startswith("gdn-b200")
    assert lib.gdn_stash_seq_floats(48, 128, 128) == 48 * 4 * 132


def _err(lib):
    return lib.gdn_last_error().decode()


def test_ba_gates_guards(lib):
    ok = dict(x=P, ks=5120, w=P, a=P, d=P, out=P, gs=96, M=4576, N=96, K=5120, nv=48, vpg=3)

    def call(**kw):
        a = {**ok, **kw}
        return lib.gdn_ba_gates(a["x"], a["ks"], a["w"], a["a"], a["d"], a["out"], a["gs"], a["M"],
                                a["N"], a["K"], a["nv"], a["vpg"], None)

    assert call(x=NULL) == _lib.GDN_ERR_NULL
    assert call(N=0, nv=0) == _lib.GDN_ERR_SHAPE and "empty BA projection" in _err(lib)
    assert call(K=5121, ks=5128) == _lib.GDN_ERR_SHAPE and "multiple of 8" in _err(lib)
    assert call(ks=5112) == _lib.GDN_ERR_STRIDE and "K_stride < K" in _err(lib)
    assert call(N=94) == _lib.GDN_ERR_SHAPE and "N != 2*nv" in _err(lib)
    assert call(vpg=5) == _lib.GDN_ERR_SHAPE
    assert call(gs=95) == _lib.GDN_ERR_STRIDE
    assert call(x=P + 8) == _lib.GDN_ERR_ALIGN
    assert call(M=0) == _lib.GDN_OK  # nothing to launch
    assert _err(lib) == ""


def test_prefill_guards(lib):
    ok = dict(q=P, k=P, qks=2048, v=P, vs=6144, g=P, b=P, gbs=48, cu=P, N=1, T=4576, h0=NULL,
              hT=NULL, o=P, Hk=16, Hv=48, dk=128, dv=128, ws=NULL, wsb=0)

    def call(**kw):
        a = {**ok, **kw}
        return lib.gdn_chunk_prefill(a["q"], a["k"], a["qks"], a["v"], a["vs"], a["g"], a["b"],
                                     a["gbs"], a["cu"], a["N"], a["T"], a["h0"], a["hT"], a["o"],
                                     a["Hk"], a["Hv"], a["dk"], a["dv"], 1.0, a["ws"], a["wsb"],
                                     None)

    assert call(q=NULL) == _lib.GDN_ERR_NULL
    assert call(cu=NULL) == _lib.GDN_ERR_NULL
    assert call(Hv=47) == _lib.GDN_ERR_SHAPE and "multiple of H_k" in _err(lib)
    assert call(dk=96, dv=96) == _lib.GDN_ERR_SHAPE
    assert call(dk=128, dv=64) == _lib.GDN_ERR_SHAPE
    assert call(N=0) == _lib.GDN_ERR_SHAPE
    assert call(qks=2040) == _lib.GDN_ERR_STRIDE
    assert call(vs=6000) == _lib.GDN_ERR_STRIDE
    assert call(gbs=47) == _lib.GDN_ERR_STRIDE
    assert call(qks=2052) == _lib.GDN_ERR_ALIGN
    assert call(o=P + 2) == _lib.GDN_ERR_ALIGN
    assert call(h0=P + 4) == _lib.GDN_ERR_ALIGN
    need = lib.gdn_chunk_prefill_workspace_bytes(4576, 1, 16, 48, 128, 128)
    if need > 0:
        assert call() == _lib.GDN_ERR_WORKSPACE


def test_verify_fold_guards(lib):
    assert lib.gdn_verify_woa(NULL, P, P, 2048, P, 6144, P, P, 48, P, P, 25344, 64, 16, 48, 128,
                              128, 1.0, P, None) == _lib.GDN_ERR_NULL
    assert "null table/stash/flag" in _err(lib)
    assert lib.gdn_verify_woa(P, P, P, 2048, P, 6144, P, P, 48, P, NULL, 25344, 64, 16, 48, 128,
                              128, 1.0, P, None) == _lib.GDN_ERR_NULL
    assert lib.gdn_verify_woa(P, P, P, 2048, P, 6144, P, P, 48, P, P, 25343, 64, 16, 48, 128,
                              128, 1.0, P, None) == _lib.GDN_ERR_SHAPE
    assert lib.gdn_verify_woa(P, P, P, 2048, P, 6144, P, P, 48, P, P, 25344, 0, 16, 48, 128,
                              128, 1.0, P, None) == _lib.GDN_OK
    assert lib.gdn_fold(P, P, P, P, 2048, NULL, 0, P, 3, 64, 16, 48, 128, 128, 25344,
                        None) == _lib.GDN_ERR_SHAPE
    assert "k_rows" in _err(lib)
    assert lib.gdn_fold(P, P, NULL, P, 2048, NULL, 0, P, 4, 64, 16, 48, 128, 128, 25344,
                        None) == _lib.GDN_ERR_NULL
    # stash and k go together; one of the two branches must have its data
    assert lib.gdn_fold(P, NULL, P, P, 2048, P, 3, P, 4, 64, 16, 48, 128, 128, 25344,
                        None) == _lib.GDN_ERR_NULL
    assert "both" in _err(lib)
    assert lib.gdn_fold(P, NULL, P, NULL, 2048, NULL, 0, P, 4, 64, 16, 48, 128, 128, 0,
                        None) == _lib.GDN_ERR_NULL
    assert "neither" in _err(lib)
    assert lib.gdn_fold(P, NULL, P, NULL, 2048, P, 2, P, 4, 64, 16, 48, 128, 128, 0,
                        None) == _lib.GDN_ERR_SHAPE
    assert "slab_entries" in _err(lib)
    assert lib.gdn_fold(P, NULL, P, NULL, 2048, P, 3, P, 4, 0, 16, 48, 128, 128, 0,
                        None) == _lib.GDN_OK
    # the parent verify: null guards, slab count, strides
    assert lib.gdn_verify_parent(NULL, P, P, 2048, P, 6144, P, P, 48, P, P, 3, 64, 16, 48, 128,
                                 128, 1.0, None) == _lib.GDN_ERR_NULL
    assert lib.gdn_verify_parent(P, P, P, 2048, P, 6144, P, P, 48, P, P, 2, 64, 16, 48, 128,
                                 128, 1.0, None) == _lib.GDN_ERR_SHAPE
    assert lib.gdn_verify_parent(P, P, P, 2047, P, 6144, P, P, 48, P, P, 3, 64, 16, 48, 128,
                                 128, 1.0, None) == _lib.GDN_ERR_STRIDE
    assert lib.gdn_verify_parent(P, P, P, 2048, P, 6144, P, P, 48, P, NULL, 0, 0, 16, 48, 128,
                                 128, 1.0, None) == _lib.GDN_OK
    assert lib.gdn_flag_clear(NULL, None) == _lib.GDN_ERR_NULL


def test_python_binding_rejects_wrong_dtypes():
    import torch
    from linear_attention_ssm_gdn_b200 import gdn_chunk_prefill
    x = torch.zeros(4, 1, 64, dtype=torch.float32)
    with pytest.raises((TypeError, ValueError)):
        gdn_chunk_prefill(x, x, x, torch.zeros(4, 1), torch.zeros(4, 1),
                          torch.tensor([0, 4], dtype=torch.int32))


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        _lib.load(str(tmp_path / "libgdn.so"))


def test_verify_static_guards(lib):
    """The no-allocation verify refuses bad arguments before it looks up its
    static stash (so no CUDA call is made here)."""
    ssf = lib.gdn_stash_seq_floats(48, 128, 128)
    assert ssf == 48 * 4 * (128 + 4)
    out = ctypes.c_void_p()

    def call(batch=64, qks=2048, vs=6144, gbs=48, Hv=48, dk=128, dv=128, stash_out=True,
             table=P, q=P):
        return lib.gdn_verify_woa_static(table, q, P, qks, P, vs, P, P, gbs, P, batch, 16, Hv, dk,
                                         dv, 1.0, P, ctypes.byref(out) if stash_out else NULL,
                                         None)

    assert call(stash_out=False) == _lib.GDN_ERR_NULL and "stash_out" in _err(lib)
    assert call(table=NULL) == _lib.GDN_ERR_NULL
    assert call(q=NULL) == _lib.GDN_ERR_NULL
    assert call(Hv=47) == _lib.GDN_ERR_SHAPE
    assert call(dk=128, dv=64) == _lib.GDN_ERR_SHAPE
    assert call(batch=-1) == _lib.GDN_ERR_SHAPE
    assert call(qks=2047) == _lib.GDN_ERR_STRIDE
    assert call(vs=6143) == _lib.GDN_ERR_STRIDE
    assert call(gbs=47) == _lib.GDN_ERR_STRIDE
    limit = (2 * 1024 * 1024) // ssf
    assert call(batch=limit + 1) == _lib.GDN_ERR_SHAPE and "exceeds the static stash" in _err(lib)


def test_verify_stride_and_shape_guards(lib):
    def call(qks=2048, vs=6144, gbs=48, batch=64, Hk=16, Hv=48, dk=128, dv=128, ssf=25344,
             stash=P):
        return lib.gdn_verify_woa(P, P, P, qks, P, vs, P, P, gbs, P, stash, ssf, batch, Hk, Hv,
                                  dk, dv, 1.0, P, None)

    assert call(qks=2047) == _lib.GDN_ERR_STRIDE
    assert call(vs=6143) == _lib.GDN_ERR_STRIDE
    assert call(gbs=47) == _lib.GDN_ERR_STRIDE
    assert call(batch=-1) == _lib.GDN_ERR_SHAPE
    assert call(Hv=40) == _lib.GDN_ERR_SHAPE  # not a multiple of H_k
    assert call(dk=96, dv=96) == _lib.GDN_ERR_SHAPE
    assert call(stash=P + 4) == _lib.GDN_ERR_ALIGN


def test_python_binding_rejects_wrong_table_and_flag_dtypes():
    """The binding checks dtypes before anything reaches the library: a float
    pointer table or engaged word is refused on the host."""
    import torch
    from linear_attention_ssm_gdn_b200 import gdn_flag_clear, gdn_fold, gdn_verify_woa
    bf = torch.zeros(4, 1, 64, dtype=torch.bfloat16)
    f = torch.zeros(4, 1, dtype=torch.float32)
    with pytest.raises(TypeError, match="h_table"):
        gdn_verify_woa(torch.zeros(1, dtype=torch.float32), bf, bf, bf, f, f,
                       torch.zeros(1, dtype=torch.int32))
    with pytest.raises(TypeError, match="h_table"):
        gdn_fold(torch.zeros(1, dtype=torch.int32), f, torch.zeros(1, dtype=torch.int32), bf,
                 torch.zeros(1, dtype=torch.int32), 1)
    with pytest.raises(TypeError, match="engaged_flag"):
        gdn_flag_clear(torch.zeros(1, dtype=torch.float32))


def test_static_stash_rejects_oversized_batch(lib):
    """gdn_verify_woa_static refuses a batch whose stash would not fit its
    static array, before any launch (so no GPU is needed)."""
    ssf = lib.gdn_stash_seq_floats(48, 128, 128)
    too_many = (2 * 1024 * 1024) // ssf + 1
    stash_ptr = ctypes.c_void_p()
    rc = lib.gdn_verify_woa_static(0x10000, 0x10000, 0x10000, 2048, 0x10000, 6144, 0x10000,
                                   0x10000, 48, 0x10000, too_many, 16, 48, 128, 128, 1.0,
                                   0x10000, ctypes.byref(stash_ptr), None)
    assert rc == _lib.GDN_ERR_SHAPE
    assert "exceeds the static stash" in lib.gdn_last_error().decode()
