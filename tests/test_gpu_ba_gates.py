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
                                        (300, 8, 4, 4), (256, 1000, 16, 1), (77, 2048, 128, 4),
                                        (40, 5120, 48, 3), (1500, 2048, 48, 3),
                                        (5000, 1024, 48, 3)])
def test_ba_gates_ragged_shapes(M, K, nv, vpg):
    """Includes 64-row tiles split 8 ways along K (M = 40), 4 ways (M = 1500)
    and 128-row tiles once 64-row pairs no longer fit the SMs (M = 5000)."""
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


@pytest.mark.parametrize("M", [1, 2, 16, 33, 64])
def test_ba_gates_decode_shapes(M):
    """Few-token (batched decode) steps at the pages' projection, N = 96,
    K = 5120: the outputs and the reduction are split across CTAs instead of
    the tokens (page "ssm_ba_gates_hopper.rs", token-count guard).  Parity at
    every element, and the time per launch is printed (CUDA events, 50
    back-to-back launches after a warm-up)."""
    ba = I.ba_inputs(M, 5120, 48, 3, seed=900 + M)
    _check(ba)
    x, w = ba.x.to(DEV), ba.w.to(DEV)
    a, dt = ba.a_log.to(DEV), ba.dt_bias.to(DEV)
    out = torch.empty(M, 96, device=DEV)
    for _ in range(5):
        gdn_ba_gates(x, w, a, dt, 3, gate_out=out)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(50):
        gdn_ba_gates(x, w, a, dt, 3, gate_out=out)
    e1.record()
    torch.cuda.synchronize()
    print(f"[timing] ba_gates M={M} N=96 K=5120: {e0.elapsed_time(e1) / 50 * 1e3:.2f} us/launch")


@pytest.mark.parametrize("M,K,nv,vpg", [(5, 8, 4, 4), (17, 40, 6, 3), (64, 200, 128, 4),
                                        (3, 2056, 2, 1)])
def test_ba_gates_decode_ragged(M, K, nv, vpg):
    """Few-token shapes with tiny or odd K (one K slice, ragged slices) and
    output counts that leave the last 8-output group partly idle."""
    _check(I.ba_inputs(M, K, nv, vpg, seed=M * 7 + K))
