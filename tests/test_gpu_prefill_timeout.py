"""The prefill's bounded waits, made to run out on purpose (no fault, no trap,
no endless loop): with a give-up time of about a microsecond, the spines'
waits for the prep CTAs' ring entries time out; the kernel must record the
timeout in its device error word, abort every CTA and return, and the next
launch with the default limit must produce exactly what a launch before the
timeout produced."""
import numpy as np
import pytest
import torch

from linear_attention_ssm_gdn_b200 import (debug_device_errors, debug_set_spin_limit,
                                           gdn_chunk_prefill)
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_prefill_wait_timeout_returns_and_recovers():
    p = I.prefill_inputs([2048, 700], 4, 8, 128, 128, seed=30, h0_std=0.02)
    d = {k: getattr(p, k).to(DEV) for k in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0")}

    def run():
        o, hT = gdn_chunk_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["cu_seqlens"],
                                  h0=d["h0"])
        torch.cuda.synchronize()
        return o.float().cpu().numpy(), hT.cpu().numpy()

    o_fresh, h_fresh = run()
    assert debug_device_errors() == [0, 0, 0, 0]
    try:
        debug_set_spin_limit(2000)  # ~1 us: far below the first ring entry's latency
        run()
        errs = debug_device_errors()
    finally:
        debug_set_spin_limit(0)
    assert errs[1] & ~64 != 0, f"no prefill timeout recorded: {errs}"
    assert errs[0] == errs[2] == errs[3] == 0, errs
    o_after, h_after = run()
    assert debug_device_errors() == [0, 0, 0, 0]
    np.testing.assert_array_equal(o_after, o_fresh)
    np.testing.assert_array_equal(h_after, h_fresh)
