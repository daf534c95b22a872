"""CPU oracle for the Gated DeltaNet hot path (f64, plain C behind ctypes).

TEST INFRASTRUCTURE ONLY: the test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the CUDA library never does.  It
shares no code with the CUDA path.

Every entry takes numpy arrays (any float dtype; they are widened to f64, so
bf16 inputs must be handed over as their exact float values) in the dense
layouts documented in ``gdn_oracle.c``:

    q, k   [T, H_k, d_k]     v, o [T, H_v, d_v]     g, beta [T, H_v]
    h0, hT [num_seqs, H_v, d_k, d_v]    (the state is H = S^T)

Sources: the pages "ssm_gdn_tc_route.rs" (prefill state spine),
"ssm_gdn_woa.rs" (K=4 verify, fold, engaged-word clear) and
"ssm_ba_gates_hopper.rs" (BA gates, ba_gates_slot); the recurrence
S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T, o_t = S_t q_t.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so with gcc (no GPU needed)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-o", tmp, _SRC,
                               "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            c_int, c_double = ctypes.c_int, ctypes.c_double
            common = [_D, _D, _D, _D, _D, _I, c_int, c_int, c_int, c_int, c_int, c_double, _D, _D, _D]
            lib.oracle_gdn_token.argtypes = common + [c_int]
            lib.oracle_gdn_chunked.argtypes = common + [c_int, c_int]
            lib.oracle_gdn_brute.argtypes = common
            lib.oracle_gdn_verify_fold.argtypes = [_D, _D, _D, _D, _D, _D, _I, _I, c_int, c_int,
                                                   c_int, c_int, c_int, c_int, c_double, _D, _D, c_int]
            lib.oracle_ba_gates.argtypes = [_D, _D, _D, _D, _D, c_int, c_int, c_int, c_int, c_int,
                                            c_int]
            for f in (lib.oracle_gdn_token, lib.oracle_gdn_chunked, lib.oracle_gdn_brute,
                      lib.oracle_gdn_verify_fold, lib.oracle_ba_gates):
                f.restype = c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(_D)


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _prefill(kind: str, q, k, v, g, beta, cu_seqlens, h0=None, scale: float = 1.0,
             chunk: int = 64, nthreads: int | None = None):
    lib = _load()
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    T, H_k, d_k = q.shape
    _, H_v, d_v = v.shape
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    num_seqs = cu.shape[0] - 1
    assert cu[0] == 0 and cu[-1] == T
    h0a = None if h0 is None else _f64(h0)
    if h0a is not None:
        assert h0a.shape == (num_seqs, H_v, d_k, d_v)
    o = np.zeros((T, H_v, d_v))
    hT = np.zeros((num_seqs, H_v, d_k, d_v))
    nt = default_threads() if nthreads is None else nthreads
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), cu.ctypes.data_as(_I), num_seqs, H_k,
            H_v, d_k, d_v, float(scale), _ptr(h0a), _ptr(o), _ptr(hT)]
    if kind == "token":
        rc = lib.oracle_gdn_token(*args, nt)
    elif kind == "chunked":
        rc = lib.oracle_gdn_chunked(*args, int(chunk), nt)
    else:
        rc = lib.oracle_gdn_brute(*args)
    if rc != 0:
        raise ValueError(f"oracle_gdn_{kind}: bad shapes")
    return o, hT


def gdn_token(q, k, v, g, beta, cu_seqlens, h0=None, scale=1.0, nthreads=None):
    """Token-by-token f64 recurrence (the definition). Returns (o, hT)."""
    return _prefill("token", q, k, v, g, beta, cu_seqlens, h0, scale, nthreads=nthreads)


def gdn_chunked(q, k, v, g, beta, cu_seqlens, h0=None, scale=1.0, chunk=64, nthreads=None):
    """Chunked WY/UT f64 form with chunk size `chunk`. Returns (o, hT)."""
    return _prefill("chunked", q, k, v, g, beta, cu_seqlens, h0, scale, chunk, nthreads)


def gdn_brute(q, k, v, g, beta, cu_seqlens, h0=None, scale=1.0):
    """Explicit transition-matrix products in long double (short sequences only)."""
    return _prefill("brute", q, k, v, g, beta, cu_seqlens, h0, scale)


def gdn_verify_fold(h_states, q, k, v, g, beta, na, present=None, K=4, scale=1.0, nthreads=None):
    """K-row verify outputs and folded states.

    h_states [batch, H_v, d_k, d_v]: each sequence's state (gathered through
    its pointer-table entry).  Rows b*K .. b*K+K-1 of q/k/v/g/beta belong to
    sequence b.  Returns (o [batch*K, H_v, d_v], h_folded like h_states).
    """
    lib = _load()
    hs = _f64(h_states)
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    batch, H_v, d_k, d_v = hs.shape
    H_k = q.shape[1]
    assert q.shape[0] == batch * K
    na_a = np.ascontiguousarray(np.asarray(na, dtype=np.int32))
    pres = np.ones(batch, dtype=np.int32) if present is None else \
        np.ascontiguousarray(np.asarray(present, dtype=np.int32))
    o = np.zeros((batch * K, H_v, d_v))
    hout = np.zeros_like(hs)
    nt = default_threads() if nthreads is None else nthreads
    rc = lib.oracle_gdn_verify_fold(_ptr(hs), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                    na_a.ctypes.data_as(_I), pres.ctypes.data_as(_I), batch, K, H_k,
                                    H_v, d_k, d_v, float(scale), _ptr(o), _ptr(hout), nt)
    if rc != 0:
        raise ValueError("oracle_gdn_verify_fold: bad shapes")
    return o, hout


def ba_gates(x, w, a_log, dt_bias, vheads_per_group, nthreads=None):
    """BA projection + gate epilogue. Returns out [M, 2*nv] = [gate | beta]."""
    lib = _load()
    x, w, a_log, dt_bias = (_f64(a) for a in (x, w, a_log, dt_bias))
    M, K = x.shape
    N = w.shape[0]
    nv = a_log.shape[0]
    out = np.zeros((M, 2 * nv))
    nt = default_threads() if nthreads is None else nthreads
    rc = lib.oracle_ba_gates(_ptr(x), _ptr(w), _ptr(a_log), _ptr(dt_bias), _ptr(out), M, N, K, nv,
                             int(vheads_per_group), nt)
    if rc != 0:
        raise ValueError("oracle_ba_gates: bad shapes")
    return out
