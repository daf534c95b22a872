"""Shared helpers for the parity tests: f64 views of the exact inputs, error
norms, and oracle runs on (sub-samples of) a workload."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances of the floating-point comparisons (bf16 operands, f32 state).
PREFILL_REL_FROB = 5e-3
PREFILL_MAX_ABS = 2e-2
BA_MAX_REL = 1e-3


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact f64 copy of a (bf16 / f32) tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def rel_frob(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def max_abs(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def oracle_prefill(q, k, v, g, beta, cu_seqlens, h0, scale=1.0, heads=None, form="token"):
    """Oracle o, hT for v-heads `heads` (all if None).

    Heads are independent, so a subset is computed exactly by giving the oracle
    only those v-heads, each with its own k-head (vpg = 1 in the sub-problem).
    Returns (o [T, len(heads), d], hT [N, len(heads), d, d]).
    """
    H_k, H_v = q.shape[1], v.shape[1]
    vpg = H_v // H_k
    heads = list(range(H_v)) if heads is None else list(heads)
    kh = [h // vpg for h in heads]
    qs, ks = f64(q)[:, kh], f64(k)[:, kh]
    vs, gs, bs = f64(v)[:, heads], f64(g)[:, heads], f64(beta)[:, heads]
    h0s = None if h0 is None else f64(h0)[:, heads]
    cu = cu_seqlens.cpu().numpy().astype(np.int32)
    fn = oracle.gdn_token if form == "token" else oracle.gdn_chunked
    return fn(qs, ks, vs, gs, bs, cu, h0s, scale)


def assert_prefill_close(o_gpu, hT_gpu, o_ref, hT_ref, what=""):
    e_o, a_o = rel_frob(o_gpu, o_ref), max_abs(o_gpu, o_ref)
    if hT_ref is not None:
        print(f"[parity] {what}: o rel_frob={e_o:.2e} max_abs={a_o:.2e}; hT rel_frob="
              f"{rel_frob(hT_gpu, hT_ref):.2e} max_abs={max_abs(hT_gpu, hT_ref):.2e}")
    assert e_o <= PREFILL_REL_FROB and a_o <= PREFILL_MAX_ABS, \
        f"{what} o: rel_frob={e_o:.3e} max_abs={a_o:.3e}"
    if hT_ref is not None:
        e_h, a_h = rel_frob(hT_gpu, hT_ref), max_abs(hT_gpu, hT_ref)
        assert e_h <= PREFILL_REL_FROB and a_h <= PREFILL_MAX_ABS, \
            f"{what} hT: rel_frob={e_h:.3e} max_abs={a_h:.3e}"
