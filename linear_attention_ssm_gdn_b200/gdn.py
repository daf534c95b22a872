"""Python binding of libgdn.so: the five hot-path calls with the C names.

Argument marshalling only: shapes and strides are read off torch tensors,
`data_ptr()`s and the current CUDA stream are passed through ctypes, and every
step of the computation runs in the library's CUDA kernels.  Outputs that the
caller does not provide are allocated here with torch (device memory is the
one thing torch is used for).  Nonzero return codes raise `GdnError` with the
name of the guard that refused.

Layouts (see include/gdn.h):
  q, k [T, H_k, d] bf16 (token stride may exceed H_k*d), v [T, H_v, d] bf16,
  g, beta [T, H_v] f32 sharing one token stride, o [T, H_v, d] bf16,
  states [N, H_v, d, d] f32 as H = S^T.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import GdnError  # noqa: F401  (re-export)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    return None if t is None else int(t.data_ptr())


def _rows(t: torch.Tensor, name: str, heads: int, d: int) -> int:
    """Token stride of a [T, heads, d] view whose (heads, d) block is dense."""
    if t.dim() != 3 or t.shape[1] != heads or t.shape[2] != d:
        raise ValueError(f"{name}: expected [T, {heads}, {d}], got {tuple(t.shape)}")
    if t.stride(2) != 1 or t.stride(1) != d:
        raise ValueError(f"{name}: the (head, dim) block must be contiguous")
    return int(t.stride(0)) if t.shape[0] > 1 else heads * d


def _need(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


def _dense(t: torch.Tensor, dtype, shape, name: str):
    """A CUDA tensor of this dtype and shape, dense in memory (the C ABI takes
    no strides for it)."""
    _need(t, dtype, name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _gates(g: torch.Tensor, beta: torch.Tensor, rows: int, H_v: int) -> int:
    """g, beta [rows, H_v] f32 with unit head stride and one shared row stride;
    returns that stride."""
    _need(g, torch.float32, "g")
    _need(beta, torch.float32, "beta")
    if tuple(g.shape) != (rows, H_v) or tuple(beta.shape) != (rows, H_v):
        raise ValueError(f"g, beta: expected [{rows}, {H_v}]")
    if H_v > 1 and (g.stride(1) != 1 or beta.stride(1) != 1):
        raise ValueError("g, beta: the head dimension must be contiguous")
    if rows > 1 and beta.stride(0) != g.stride(0):
        raise ValueError("g and beta must share one row stride")
    return int(g.stride(0)) if rows > 1 else H_v


def version() -> str:
    return _lib.load().gdn_version().decode()


def gdn_ba_gates(x, w_ba, a_log, dt_bias, vheads_per_group, gate_out=None, stream=None):
    """BA projection + gates. x [M, K] (row stride >= K) bf16, w_ba [2 nv, K] bf16,
    a_log/dt_bias [nv] f32 -> gate_out [M, 2 nv] f32 = [gate | beta]."""
    lib = _lib.load()
    _need(x, torch.bfloat16, "x")
    _need(w_ba, torch.bfloat16, "w_ba")
    M, K = x.shape
    N = w_ba.shape[0]
    nv = a_log.shape[0]
    if x.stride(1) != 1 or not w_ba.is_contiguous():
        raise ValueError("x rows and w_ba must be dense along K")
    _dense(a_log, torch.float32, (nv,), "a_log")
    _dense(dt_bias, torch.float32, (nv,), "dt_bias")
    if gate_out is None:
        gate_out = torch.empty(M, 2 * nv, dtype=torch.float32, device=x.device)
    _need(gate_out, torch.float32, "gate_out")
    if gate_out.dim() != 2 or gate_out.shape[0] != M or gate_out.shape[1] < 2 * nv or \
            (2 * nv > 1 and gate_out.stride(1) != 1):
        raise ValueError(f"gate_out: expected [{M}, >= {2 * nv}] with contiguous rows")
    k_stride = int(x.stride(0)) if M > 1 else K
    rc = lib.gdn_ba_gates(_ptr(x), k_stride, _ptr(w_ba), _ptr(a_log), _ptr(dt_bias),
                          _ptr(gate_out), int(gate_out.stride(0)), M, N, K, nv,
                          int(vheads_per_group), _stream(stream))
    _lib.check("gdn_ba_gates", rc)
    return gate_out


def gdn_chunk_prefill_workspace_bytes(total_tokens, num_seqs, H_k, H_v, d_k, d_v) -> int:
    return int(_lib.load().gdn_chunk_prefill_workspace_bytes(total_tokens, num_seqs, H_k, H_v,
                                                             d_k, d_v))


def gdn_chunk_prefill(q, k, v, g, beta, cu_seqlens, h0=None, hT=None, o=None, scale=1.0,
                      workspace=None, store_final_state=True, stream=None, limbs=1,
                      segments=None):
    """Chunked prefill over packed sequences. Returns (o, hT).  limbs=2 calls
    gdn_chunk_prefill_x2 (the state enters the MMAs as two bf16 limbs);
    segments=S calls gdn_chunk_prefill_segmented (two-level scan with S
    segments per sequence; None lets the library choose)."""
    lib = _lib.load()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(g, torch.float32, "g")
    _need(beta, torch.float32, "beta")
    T, H_k, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    qk_stride = _rows(q, "q", H_k, d_k)
    if _rows(k, "k", H_k, d_k) != qk_stride:
        raise ValueError("q and k must share one token stride")
    v_stride = _rows(v, "v", H_v, d_v)
    gb_stride = _gates(g, beta, T, H_v)
    _need(cu_seqlens, torch.int32, "cu_seqlens")
    num_seqs = cu_seqlens.shape[0] - 1
    if o is None:
        o = torch.empty(T, H_v, d_v, dtype=torch.bfloat16, device=q.device)
    _dense(o, torch.bfloat16, (T, H_v, d_v), "o")
    if hT is None and store_final_state:
        hT = torch.empty(num_seqs, H_v, d_k, d_v, dtype=torch.float32, device=q.device)
    for t, n in ((h0, "h0"), (hT, "hT")):
        if t is not None:
            _dense(t, torch.float32, (num_seqs, H_v, d_k, d_v), n)
    if segments is None:
        need = int(lib.gdn_chunk_prefill_workspace_bytes(T, num_seqs, H_k, H_v, d_k, d_v))
    else:
        need = int(lib.gdn_chunk_prefill_segmented_workspace_bytes(T, num_seqs, H_k, H_v, d_k,
                                                                   d_v, int(segments)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace is not None and not workspace.is_cuda:
        raise ValueError("workspace: must be a CUDA tensor")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if limbs not in (1, 2):
        raise ValueError("limbs must be 1 or 2")
    args = (_ptr(q), _ptr(k), qk_stride, _ptr(v), v_stride, _ptr(g), _ptr(beta), gb_stride,
            _ptr(cu_seqlens), num_seqs, T, _ptr(h0), _ptr(hT), _ptr(o), H_k, H_v, d_k, d_v,
            float(scale))
    if segments is None:
        name = "gdn_chunk_prefill" if limbs == 1 else "gdn_chunk_prefill_x2"
        rc = getattr(lib, name)(*args, _ptr(workspace), ws_bytes, _stream(stream))
    else:
        name = "gdn_chunk_prefill_segmented"
        rc = lib.gdn_chunk_prefill_segmented(*args, int(segments), int(limbs), _ptr(workspace),
                                             ws_bytes, _stream(stream))
    _lib.check(name, rc)
    return o, hT


def gdn_stash_seq_floats(H_v, d_k, d_v) -> int:
    return int(_lib.load().gdn_stash_seq_floats(H_v, d_k, d_v))


def gdn_verify_woa(h_table, q, k, v, g, beta, engaged_flag, o=None, stash=None, scale=1.0,
                   stream=None):
    """K=4 verify. h_table: int64 CUDA tensor [batch] of state pointers.
    Returns (o [batch*4, H_v, d] bf16, stash f32 [batch, stash_seq_floats])."""
    lib = _lib.load()
    _need(h_table, torch.int64, "h_table")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    _need(engaged_flag, torch.int32, "engaged_flag")
    R, H_k, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    batch = h_table.shape[0]
    if R != 4 * batch:
        raise ValueError("q/k/v must hold 4 rows per sequence")
    qk_stride = _rows(q, "q", H_k, d_k)
    if _rows(k, "k", H_k, d_k) != qk_stride:
        raise ValueError("q and k must share one row stride")
    v_stride = _rows(v, "v", H_v, d_v)
    gb_stride = _gates(g, beta, R, H_v)
    ssf = gdn_stash_seq_floats(H_v, d_k, d_v)
    if o is None:
        o = torch.empty(R, H_v, d_v, dtype=torch.bfloat16, device=q.device)
    _dense(o, torch.bfloat16, (R, H_v, d_v), "o")
    if stash is None:
        stash = torch.empty(batch, ssf, dtype=torch.float32, device=q.device)
    _need(stash, torch.float32, "stash")
    if stash.dim() != 2 or stash.shape[0] != batch or stash.shape[1] < ssf or \
            (ssf > 1 and stash.stride(1) != 1):
        raise ValueError(f"stash: expected [{batch}, >= {ssf}] with contiguous rows")
    rc = lib.gdn_verify_woa(_ptr(h_table), _ptr(q), _ptr(k), qk_stride, _ptr(v), v_stride,
                            _ptr(g), _ptr(beta), gb_stride, _ptr(o), _ptr(stash),
                            int(stash.stride(0)) if batch > 1 else ssf, batch, H_k, H_v, d_k,
                            d_v, float(scale), _ptr(engaged_flag), _stream(stream))
    _lib.check("gdn_verify_woa", rc)
    return o, stash


def _slab_table(hi_tables, batch):
    """hi_tables: int64 CUDA tensor [batch, slab_entries] of state pointers (or None)."""
    if hi_tables is None:
        return None, 0
    _need(hi_tables, torch.int64, "hi_tables")
    if hi_tables.dim() != 2 or hi_tables.shape[0] != batch or not hi_tables.is_contiguous():
        raise ValueError(f"hi_tables: expected a contiguous [{batch}, slab_entries] table")
    return _ptr(hi_tables), int(hi_tables.shape[1])


def gdn_verify_parent(h_table, q, k, v, g, beta, hi_tables=None, o=None, scale=1.0,
                      stream=None):
    """Parent K=4 verify: outputs as gdn_verify_woa; the states after rows 0..2
    go to the slabs hi_tables[b, r] (int64 [batch, slab_entries] table of state
    pointers), the state after row 3 replaces the live state.  Returns o."""
    lib = _lib.load()
    _need(h_table, torch.int64, "h_table")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    R, H_k, d_k = q.shape
    H_v, d_v = v.shape[1], v.shape[2]
    batch = h_table.shape[0]
    if R != 4 * batch:
        raise ValueError("q/k/v must hold 4 rows per sequence")
    qk_stride = _rows(q, "q", H_k, d_k)
    if _rows(k, "k", H_k, d_k) != qk_stride:
        raise ValueError("q and k must share one row stride")
    v_stride = _rows(v, "v", H_v, d_v)
    gb_stride = _gates(g, beta, R, H_v)
    if o is None:
        o = torch.empty(R, H_v, d_v, dtype=torch.bfloat16, device=q.device)
    _dense(o, torch.bfloat16, (R, H_v, d_v), "o")
    hp, se = _slab_table(hi_tables, batch)
    rc = lib.gdn_verify_parent(_ptr(h_table), _ptr(q), _ptr(k), qk_stride, _ptr(v), v_stride,
                               _ptr(g), _ptr(beta), gb_stride, _ptr(o), hp, se, batch, H_k, H_v,
                               d_k, d_v, float(scale), _stream(stream))
    _lib.check("gdn_verify_parent", rc)
    return o


def gdn_fold(h_table, stash, na_tab, k, engaged_flag, H_v, k_rows=4, hi_tables=None,
             stream=None):
    """Post-verdict fold: each state ends as the state after its first
    na_tab[b] verified rows -- by applying the write-on-accept stash (engaged
    word set) or by restoring a parent verify's slab (engaged word clear;
    hi_tables as passed to gdn_verify_parent).  stash may be None when only the
    parent path is used; k is always given (its shape fixes H_k and d)."""
    lib = _lib.load()
    _need(h_table, torch.int64, "h_table")
    _need(k, torch.bfloat16, "k")
    _need(engaged_flag, torch.int32, "engaged_flag")
    batch = h_table.shape[0]
    _dense(na_tab, torch.int32, (batch,), "na_tab")
    _, H_k, d = k.shape
    qk_stride = _rows(k, "k", H_k, d)
    if stash is not None:
        _need(stash, torch.float32, "stash")
        ssf = int(stash.stride(0)) if batch > 1 else gdn_stash_seq_floats(H_v, d, d)
        k_ptr = _ptr(k)
    else:
        ssf, k_ptr = 0, None
    hp, se = _slab_table(hi_tables, batch)
    rc = lib.gdn_fold(_ptr(h_table), _ptr(stash), _ptr(na_tab), k_ptr, qk_stride, hp, se,
                      _ptr(engaged_flag), int(k_rows), batch, H_k, H_v, d, d, ssf,
                      _stream(stream))
    _lib.check("gdn_fold", rc)


def gdn_flag_clear(engaged_flag, stream=None):
    _need(engaged_flag, torch.int32, "engaged_flag")
    rc = _lib.load().gdn_flag_clear(_ptr(engaged_flag), _stream(stream))
    _lib.check("gdn_flag_clear", rc)


def debug_device_errors() -> list[int]:
    """Read and clear the library's device error words (synchronises)."""
    out = (ctypes.c_uint32 * 4)()
    rc = _lib.load().gdn_debug_device_errors(ctypes.addressof(out))
    _lib.check("gdn_debug_device_errors", rc)
    return list(out)


def debug_set_spin_limit(cycles: int) -> None:
    """Give-up time (clock cycles) of the prefill's pipeline waits for the
    launches that follow; 0 restores the default (about 2 s).  Diagnostics."""
    rc = _lib.load().gdn_debug_set_spin_limit(int(cycles))
    _lib.check("gdn_debug_set_spin_limit", rc)
