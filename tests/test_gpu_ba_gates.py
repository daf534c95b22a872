"""GPU parity of gdn_ba_gates (through the C ABI) against the f64 oracle:
max elementwise relative error <= 1e-3 on every gate and beta."""
import numpy as np
import pytest
import torch

import oracle
from helpers import BA_MAX_REL, f64
from linear_attention_ssm_gdn_b200 import debug_device_errors, gdn_ba_gates
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(ba: I.BAInputs, x_dev=None):
    x = ba.x.to(DEV) if x_dev is None else x_dev
    out = gdn_ba_gates(x, ba.w.to(DEV), ba.a_log.to(DEV), ba.dt_bias.to(DEV),
                       ba.vheads_per_group)
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    ref = oracle.ba_gates(f64(ba.x), f64(ba.w), f64(ba.a_log), f64(ba.dt_bias),
                          ba.vheads_per_group)
    got = out.cpu().numpy().astype(np.float64)
    rel = np.abs(got - ref) / np.abs(ref)
    assert float(rel.max()) <= BA_MAX_REL, f"max rel err {rel.max():.3e}"
    return got


def test_ba_gates_full_size_4576x5120():
    _check(I.workload(2).ba)


@pytest.mark.parametrize("M,K,nv,vpg", [(1, 5120, 48, 3), (100, 64, 6, 3), (129, 72, 8, 2),
                                        (300, 8, 4, 4), (256, 1000, 16, 1), (77, 2048, 128, 4)])
def test_ba_gates_ragged_shapes(M, K, nv, vpg):
    _check(I.ba_inputs(M, K, nv, vpg, seed=M + K))


def test_ba_gates_strided_rows_and_output():
    ba = I.ba_inputs(200, 512, 48, 3, seed=3)
    wide = torch.zeros(200, 512 + 64, dtype=torch.bfloat16)
    wide[:, :512] = ba.x
    x = wide.to(DEV)[:, :512]
    assert x.stride(0) == 576
    _check(ba, x_dev=x)
    out = torch.full((200, 100), 7.0, device=DEV)
    gdn_ba_gates(ba.x.to(DEV), ba.w.to(DEV), ba.a_log.to(DEV), ba.dt_bias.to(DEV), 3,
                 gate_out=out[:, :96])
    torch.cuda.synchronize()
    assert torch.all(out[:, 96:] == 7.0)  # the padding columns are never written


def test_ba_gates_zero_weight_closed_form():
    ba = I.ba_inputs(130, 256, 6, 3, seed=4)
    ba.w = torch.zeros_like(ba.w)
    got = _check(ba)
    want_g = -np.exp(f64(ba.a_log)) * np.log1p(np.exp(f64(ba.dt_bias)))
    np.testing.assert_allclose(got[:, :6], np.broadcast_to(want_g, (130, 6)), rtol=1e-5)
    np.testing.assert_allclose(got[:, 6:], 0.5, rtol=1e-6)


def test_ba_gates_wide_range():
    """Weights scaled so that |ba| reaches about 60: softplus runs through both
    of its branches (series for e^{-|z|} < 1/16, logarithm above) and the
    sigmoid through its tails; every output within the elementwise bound."""
    ba = I.ba_inputs(512, 1024, 48, 3, seed=5)
    ba.w = (ba.w.float() * 20.0).to(torch.bfloat16)
    got = _check(ba)
    assert float(np.abs(got[:, :48]).min()) < 1e-6 < float(np.abs(got[:, :48]).max())
