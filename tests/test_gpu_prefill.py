"""GPU parity of gdn_chunk_prefill (through the C ABI) against the f64 oracle.

Small cases are compared element by element over every head; the full-size
workloads (4096 and 4576 tokens, 8 ragged sequences) on a sample of v-heads
that the oracle recomputes exactly.  Tolerances: relative Frobenius <= 5e-3
and max-abs <= 2e-2 on o and hT (bf16 operands, f32 state).
"""
import numpy as np
import pytest
import torch

from helpers import assert_prefill_close, f64, oracle_prefill
from linear_attention_ssm_gdn_b200 import debug_device_errors, gdn_ba_gates, gdn_chunk_prefill
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _to_dev(p: I.PrefillInputs):
    return {k: (getattr(p, k).to(DEV) if getattr(p, k) is not None else None)
            for k in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0")}


def _run(p, h0=True, scale=1.0, **kw):
    d = _to_dev(p)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                              h0=d["h0"] if h0 else None, scale=scale, **kw)
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    return o.float().cpu().numpy(), hT.cpu().numpy()


def _check(p, heads=None, h0=True, scale=1.0, what=""):
    o, hT = _run(p, h0=h0, scale=scale)
    o_ref, hT_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens,
                                   p.h0 if h0 else None, scale, heads)
    if heads is not None:
        o, hT = o[:, heads], hT[:, heads]
    assert_prefill_close(o, hT, o_ref, hT_ref, what)


def test_tiny_workload_d64():
    """T=256, H_k=H_v=2, d=64, h0 = 0 (every head, every element)."""
    _check(I.workload(0).prefill, what="tiny")


@pytest.mark.parametrize("seqlens", [[64], [1], [63], [65], [200], [1, 63, 64, 65, 130, 7]])
def test_ragged_lengths_d128(seqlens):
    """Several chunks and ragged tails: 1, 63, 64, 65, 130 rows; GQA 2 -> 4 heads."""
    p = I.prefill_inputs(seqlens, 2, 4, 128, 128, seed=11, h0_std=0.02)
    _check(p, what=str(seqlens))


def test_zero_initial_state_null_h0():
    p = I.prefill_inputs([150, 90], 1, 2, 128, 128, seed=12, h0_std=None)
    _check(p, h0=False, what="h0=None")


def test_empty_sequences_copy_state():
    """Length-0 sequences (first, middle, last) keep h0 as hT and emit no rows."""
    p = I.prefill_inputs([0, 100, 0, 70, 0], 2, 2, 128, 128, seed=13, h0_std=0.05)
    _check(p, what="empty seqs")
    _, hT = _run(p)
    h0 = p.h0.numpy()
    for n in (0, 2, 4):
        np.testing.assert_array_equal(hT[n], h0[n])


def test_scale_and_positive_scale():
    p = I.prefill_inputs([129], 1, 1, 128, 128, seed=14, h0_std=0.02)
    _check(p, scale=0.088388, what="scale")


def test_strided_views_and_inplace_state():
    """q/k/v as views into wider rows; g/beta as column blocks of one [T, 2H] tensor;
    hT written in place over h0."""
    T, H_k, H_v, d = 300, 2, 4, 128
    p = I.prefill_inputs([120, 180], H_k, H_v, d, d, seed=15, h0_std=0.02)
    qk = torch.zeros(T, 2 * H_k * d + 64, dtype=torch.bfloat16)
    qk[:, :H_k * d] = p.q.reshape(T, -1)
    qk[:, H_k * d + 64:] = p.k.reshape(T, -1)
    vv = torch.zeros(T, H_v * d + 128, dtype=torch.bfloat16)
    vv[:, 128:] = p.v.reshape(T, -1)
    gb = torch.zeros(T, 2 * H_v + 3)
    gb[:, :H_v] = p.g
    gb[:, H_v + 3:] = p.beta
    qk_d, vv_d, gb_d = qk.to(DEV), vv.to(DEV), gb.to(DEV)
    q = qk_d[:, :H_k * d].view(T, H_k, d)
    k = qk_d[:, H_k * d + 64:].view(T, H_k, d)
    v = vv_d[:, 128:].view(T, H_v, d)
    g, beta = gb_d[:, :H_v], gb_d[:, H_v + 3:]
    h = p.h0.to(DEV).clone()
    o, hT = gdn_chunk_prefill(q, k, v, g, beta, p.cu_seqlens.to(DEV), h0=h, hT=h)
    torch.cuda.synchronize()
    assert hT.data_ptr() == h.data_ptr()
    o_ref, hT_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, p.h0)
    assert_prefill_close(o.float().cpu().numpy(), h.cpu().numpy(), o_ref, hT_ref, "strided")


def test_single_sequence_4096_tokens_sampled_heads():
    """T=4096, H_k=16, H_v=32, d=128, h0 ~ N(0, 0.02): heads 0, 1, 17, 31."""
    _check(I.workload(1).prefill, heads=[0, 1, 17, 31], what="T=4096")


def test_ba_front_end_4576_tokens_sampled_heads():
    """M=4576: g, beta from gdn_ba_gates (GPU) vs the oracle's own BA gates."""
    import oracle
    w = I.workload(2)
    p, ba = w.prefill, w.ba
    gates = gdn_ba_gates(ba.x.to(DEV), ba.w.to(DEV), ba.a_log.to(DEV), ba.dt_bias.to(DEV),
                         ba.vheads_per_group)
    nv = ba.nv
    d = _to_dev(p)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], gates[:, :nv], gates[:, nv:],
                              d["cu_seqlens"], h0=d["h0"])
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    gref = oracle.ba_gates(f64(ba.x), f64(ba.w), f64(ba.a_log), f64(ba.dt_bias),
                           ba.vheads_per_group)
    heads = [0, 5, 23, 47]
    o_ref, hT_ref = oracle_prefill(p.q, p.k, p.v, torch.from_numpy(gref[:, :nv]),
                                   torch.from_numpy(gref[:, nv:]), p.cu_seqlens, p.h0, 1.0, heads)
    assert_prefill_close(o.float().cpu().numpy()[:, heads], hT.cpu().numpy()[:, heads], o_ref,
                         hT_ref, "M=4576")


def test_varlen_8_sequences_sampled_heads():
    """8 sequences of 512..8192 tokens (packed, 24,674 tokens as drawn), heads 2 and 40."""
    _check(I.workload(3).prefill, heads=[2, 40], what="varlen")


def test_strong_decay_gates_stay_finite():
    """Gates down to -15 per token (chunk decay ~ e^-600) keep o and hT finite and exact."""
    p = I.prefill_inputs([140], 1, 1, 128, 128, seed=16, h0_std=0.02)
    p.g = -torch.rand(p.g.shape, generator=torch.Generator().manual_seed(5)) * 15.0
    o, hT = _run(p)
    assert np.isfinite(o).all() and np.isfinite(hT).all()
    _check(p, what="strong decay")


def test_repeat_calls_are_deterministic():
    p = I.prefill_inputs([333], 2, 4, 128, 128, seed=17, h0_std=0.02)
    o1, h1 = _run(p)
    o2, h2 = _run(p)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(h1, h2)


def test_positive_gates_within_the_bound_are_exact():
    """Gates of both signs, g ~ N(-0.1, 0.15) (up to +0.3 per token): the
    cumulative gate rises and falls within each chunk by far less than the
    documented bound of 80, so every decay factor stays finite and the result
    matches the oracle.  (Gates that make the state grow for many chunks, e.g.
    N(0, 0.3) with a 3000-fold growth, cost precision like weak decay does --
    5.4e-3 there, on the GPU and in a rounding-exact CPU emulation alike.)"""
    p = I.prefill_inputs([700, 130], 1, 2, 128, 128, seed=20, h0_std=0.02)
    p.g = torch.randn(p.g.shape, generator=torch.Generator().manual_seed(21)) * 0.15 - 0.1
    assert float(p.g.max()) > 0.25
    _check(p, what="positive gates")


def test_gate_rise_beyond_the_bound_is_flagged():
    """A chunk whose cumulative gate rises by more than 80 (g = +2 on all 64
    rows: a rise of 128) cannot be represented by the f32 decay factors: the
    prefill sets bit 64 of its device error word instead of returning silent
    garbage (its outputs are undefined and not compared)."""
    p = I.prefill_inputs([64], 1, 1, 128, 128, seed=22, h0_std=None)
    p.g = torch.full(p.g.shape, 2.0)
    d = _to_dev(p)
    gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"])
    torch.cuda.synchronize()
    errs = debug_device_errors()
    assert errs[1] == 64 and errs[0] == errs[2] == errs[3] == 0, errs
    # the flag does not stick: a normal call afterwards reports nothing
    _check(I.prefill_inputs([64], 1, 1, 128, 128, seed=23, h0_std=None), what="after flag")
