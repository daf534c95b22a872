"""GPU parity of the segment-parallel (two-level) prefill scan, through the C ABI
(gdn_chunk_prefill_segmented; gdn_chunk_prefill takes the same path on its own
for few (sequence, head) units).

Against the f64 oracle with the prefill tolerances, for 2 .. 8 segments per
sequence: ragged and empty sequences, no initial state, an in-place final
state, weak decay with a large initial state (where every segment's
transition matters), and the two-limb spine.  The timing test prints the
single-level and two-level launch times on a tensor-parallel-sized shard of
the pages' geometry (6 v-heads) over a 16384-token sequence.
"""
import numpy as np
import pytest
import torch

from helpers import assert_prefill_close, oracle_prefill
from linear_attention_ssm_gdn_b200 import _lib, debug_device_errors, gdn_chunk_prefill
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(p):
    return {k: (getattr(p, k).to(DEV) if getattr(p, k) is not None else None)
            for k in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0")}


def _run(p, segments, h0=True, limbs=1, **kw):
    d = _dev(p)
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                              h0=d["h0"] if h0 else None, segments=segments, limbs=limbs, **kw)
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    return o.float().cpu().numpy(), hT.cpu().numpy()


@pytest.mark.parametrize("segments", [2, 3, 4, 8])
def test_segmented_tp_shard(segments):
    """4576 tokens, H_k = 2, H_v = 6 (the pages' geometry over 8 GPUs), h0 ~ N(0, 0.02)."""
    p = I.prefill_inputs([4576], 2, 6, 128, 128, seed=80, h0_std=0.02)
    o, hT = _run(p, segments)
    o_ref, h_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, p.h0)
    assert_prefill_close(o, hT, o_ref, h_ref, f"segments={segments}")


def test_segmented_varlen_empty_and_no_h0():
    """Ragged sequences, empty ones among them (first, middle, last), h0 = NULL:
    segments of different lengths per sequence, empty segments, short tails."""
    p = I.prefill_inputs([0, 700, 65, 0, 1300, 1, 0], 1, 3, 128, 128, seed=81, h0_std=None)
    o, hT = _run(p, 5, h0=False)
    o_ref, h_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, None)
    assert_prefill_close(o, hT, o_ref, h_ref, "varlen segments=5")
    for n in (0, 3, 6):
        assert np.all(hT[n] == 0)


def test_segmented_in_place_state_d64():
    p = I.prefill_inputs([900, 333], 2, 4, 64, 64, seed=82, h0_std=0.05)
    d = _dev(p)
    h = d["h0"].clone()
    o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"], h0=h,
                              hT=h, segments=4)
    torch.cuda.synchronize()
    assert hT.data_ptr() == h.data_ptr()
    o_ref, h_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, p.h0)
    assert_prefill_close(o.float().cpu().numpy(), h.cpu().numpy(), o_ref, h_ref,
                         "in place d=64 segments=4")


@pytest.mark.parametrize("limbs", [1, 2])
def test_segmented_weak_decay_large_state(limbs):
    """g = log-sigmoid(N(6, 1)) (the state remembers hundreds of tokens, so each
    segment's transition M is far from zero) and h0 ~ N(0, 1)."""
    p = I.prefill_inputs([4096], 1, 2, 128, 128, seed=83, h0_std=1.0)
    gen = torch.Generator().manual_seed(84)
    p.g = torch.nn.functional.logsigmoid(torch.randn(p.g.shape, generator=gen) + 6.0)
    o, hT = _run(p, 8, limbs=limbs)
    o_ref, h_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, p.h0)
    assert_prefill_close(o, hT, o_ref, h_ref, f"weak decay segments=8 limbs={limbs}")


def test_segmented_matches_single_level_and_is_chosen_for_few_heads():
    """The library picks two levels on its own for few units (workspace query
    and call agree), and the result matches the single-level scan within the
    tolerances; the two launch times are printed."""
    lib = _lib.load()
    T, H_k, H_v = 16384, 2, 6
    auto = int(lib.gdn_chunk_prefill_workspace_bytes(T, 1, H_k, H_v, 128, 128))
    single = int(lib.gdn_chunk_prefill_segmented_workspace_bytes(T, 1, H_k, H_v, 128, 128, 1))
    assert auto > single  # the per-segment states live in the workspace
    p = I.prefill_inputs([T], H_k, H_v, 128, 128, seed=85, h0_std=0.02)
    d = _dev(p)
    times = {}
    outs = {}
    for name, seg in (("single", 1), ("auto", None)):
        o = torch.empty(T, H_v, 128, dtype=torch.bfloat16, device=DEV)
        hT = torch.empty_like(d["h0"])
        call = lambda: gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"],
                                         d["cu_seqlens"], h0=d["h0"], hT=hT, o=o,
                                         segments=seg)
        for _ in range(3):
            call()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(10):
            call()
        e1.record()
        torch.cuda.synchronize()
        times[name] = e0.elapsed_time(e1) / 10 * 1e3
        outs[name] = (o.float().cpu().numpy(), hT.cpu().numpy())
    print(f"[timing] prefill T={T} H_k={H_k} H_v={H_v}: single-level {times['single']:.1f} us, "
          f"two-level (auto) {times['auto']:.1f} us")
    assert_prefill_close(outs["auto"][0], outs["auto"][1], outs["single"][0], outs["single"][1],
                         "auto vs single")
