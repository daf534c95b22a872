"""The one-limb (gdn_chunk_prefill) and two-limb (gdn_chunk_prefill_x2) state
spines side by side (page "ssm_gdn_tc_route.rs": _tcfuse vs _tcfuse_x2).

Both must meet the prefill tolerances against the f64 oracle on the same
inputs; the printed [limbs] lines record their errors, including a stress
case (T = 8192, weak decay, large initial state) where the state's rounding
matters most.
"""
import numpy as np
import pytest
import torch

from helpers import assert_prefill_close, max_abs, oracle_prefill, rel_frob
from linear_attention_ssm_gdn_b200 import debug_device_errors, gdn_chunk_prefill
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(p, heads, what):
    d = {k: getattr(p, k).to(DEV) for k in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0")}
    o_ref, h_ref = oracle_prefill(p.q, p.k, p.v, p.g, p.beta, p.cu_seqlens, p.h0, 1.0, heads)
    errs = {}
    for limbs in (1, 2):
        o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                  h0=d["h0"], limbs=limbs)
        torch.cuda.synchronize()
        assert debug_device_errors() == [0, 0, 0, 0]
        o = o.float().cpu().numpy()[:, heads]
        hT = hT.cpu().numpy()[:, heads]
        assert_prefill_close(o, hT, o_ref, h_ref, f"{what} limbs={limbs}")
        errs[limbs] = (rel_frob(o, o_ref), max_abs(o, o_ref), rel_frob(hT, h_ref))
    for limbs, (eo, ao, eh) in errs.items():
        print(f"[limbs] {what} limbs={limbs}: o rel_frob={eo:.3e} max_abs={ao:.2e} "
              f"hT rel_frob={eh:.3e}")
    return errs


def test_limbs_single_sequence_4096():
    _both(I.workload(1).prefill, [0, 1, 17, 31], "T=4096 H 16/32")


def test_limbs_4576_tokens_48_heads():
    p = I.prefill_inputs([4576], 16, 48, 128, 128, seed=2, h0_std=None)
    _both(p, [0, 5, 23, 47], "T=4576 H 16/48")


def test_limbs_varlen():
    _both(I.workload(3).prefill, [2, 40], "varlen 8 seqs")


def test_limbs_weak_decay_long_large_state():
    """T = 8192, g = log-sigmoid(N(9, 1)) (decay ~ 1e-4 per token: the state
    remembers thousands of tokens), h0 ~ N(0, 1)."""
    p = I.prefill_inputs([8192], 1, 2, 128, 128, seed=6, h0_std=1.0)
    gen = torch.Generator().manual_seed(66)
    p.g = torch.nn.functional.logsigmoid(torch.randn(p.g.shape, generator=gen) + 9.0)
    _both(p, [0, 1], "T=8192 weak decay h0~N(0,1)")


@pytest.mark.parametrize("seqlens", [[1, 63, 64, 65, 130]])
def test_limbs_ragged_d64(seqlens):
    p = I.prefill_inputs(seqlens, 1, 3, 64, 64, seed=19, h0_std=0.05)
    _both(p, [0, 1, 2], "ragged d=64")
