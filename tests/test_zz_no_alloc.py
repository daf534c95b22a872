"""gdn_verify_woa_static: the verify for callers that cannot allocate.

Some callers of this library cannot allocate device memory themselves: an
engine that reserved all of it up front in its own pool, or a decode loop that
must never call cudaMalloc because it can stall the whole device.  For them
the verify's stash (the scratch it leaves for the fold) lives in a static
array inside the library.  This test calls that entry point through the C ABI
twice in a row, on two different inputs, and checks that its outputs, and the
fold driven by the stash address it hands back, match the regular
gdn_verify_woa path on the same inputs.  (The refusal of an oversized batch
needs no GPU and is tested with the other guards in test_abi.py.)

The file name makes pytest collect it last; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import PREFILL_MAX_ABS, PREFILL_REL_FROB, max_abs, rel_frob
from linear_attention_ssm_gdn_b200 import _lib, gdn_flag_clear, gdn_fold, gdn_verify_woa
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _prepare(vi):
    pool = vi.pool.to(DEV).clone()
    per = pool[0].numel() * 4
    table = torch.tensor([pool.data_ptr() + int(s) * per for s in vi.slots], dtype=torch.int64,
                         device=DEV)
    d = {k: getattr(vi, k).to(DEV) for k in ("q", "k", "v", "g", "beta", "na")}
    return pool, table, d


def _static_verify(lib, table, d, vi, o, flag):
    stash_ptr = ctypes.c_void_p()
    stream = torch.cuda.current_stream().cuda_stream
    H_k, H_v, dk = vi.H_k, vi.H_v, vi.d_k
    rc = lib.gdn_verify_woa_static(
        table.data_ptr(), d["q"].data_ptr(), d["k"].data_ptr(), H_k * dk, d["v"].data_ptr(),
        H_v * vi.d_v, d["g"].data_ptr(), d["beta"].data_ptr(), H_v, o.data_ptr(), vi.batch, H_k,
        H_v, dk, vi.d_v, 1.0, flag.data_ptr(), ctypes.byref(stash_ptr), stream)
    assert rc == 0, lib.gdn_last_error().decode()
    assert stash_ptr.value
    return stash_ptr.value


def _regular(vi):
    """Verify + fold through the regular entry point (caller-allocated stash)."""
    pool, table, d = _prepare(vi)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn_flag_clear(flag)
    o, stash = gdn_verify_woa(table, d["q"], d["k"], d["v"], d["g"], d["beta"], flag)
    gdn_fold(table, stash, d["na"], d["k"], flag, vi.H_v)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), pool.cpu().numpy()


def test_static_stash_verify_matches_regular_twice():
    lib = _lib.load()
    # Two calls in a row on DIFFERENT inputs (another seed, so other states,
    # rows and accepted counts): the second call must replace the shared
    # array's contents, not reuse what the first call left there.
    first = I.workload(4).verify  # batch 64 x 4 rows, 48 heads, d = 128
    second = I.verify_inputs(64, 4, 16, 48, 128, 128, slots_total=128, seed=104)
    assert not torch.equal(first.na, second.na)
    for call, vi in enumerate((first, second)):
        ssf = lib.gdn_stash_seq_floats(vi.H_v, vi.d_k, vi.d_v)
        assert vi.batch * ssf <= 2 * 1024 * 1024
        o_ref, pool_ref = _regular(vi)

        pool, table, d2 = _prepare(vi)
        flag = torch.zeros(1, dtype=torch.int32, device=DEV)
        gdn_flag_clear(flag)
        o = torch.empty(vi.batch * 4, vi.H_v, vi.d_v, dtype=torch.bfloat16, device=DEV)
        stash_addr = _static_verify(lib, table, d2, vi, o, flag)
        rc = lib.gdn_fold(table.data_ptr(), stash_addr, d2["na"].data_ptr(), d2["k"].data_ptr(),
                          vi.H_k * vi.d_k, None, 0, flag.data_ptr(), 4, vi.batch, vi.H_k, vi.H_v,
                          vi.d_k, vi.d_v, ssf, torch.cuda.current_stream().cuda_stream)
        assert rc == 0, lib.gdn_last_error().decode()
        torch.cuda.synchronize()
        o_np = o.float().cpu().numpy()
        p_np = pool.cpu().numpy()
        assert int(flag.item()) == 1, f"call {call}: engaged word {int(flag.item())}"
        assert rel_frob(o_np, o_ref) <= PREFILL_REL_FROB and \
            max_abs(o_np, o_ref) <= PREFILL_MAX_ABS, f"call {call}: verify outputs differ"
        assert rel_frob(p_np, pool_ref) <= PREFILL_REL_FROB and \
            max_abs(p_np, pool_ref) <= PREFILL_MAX_ABS, f"call {call}: folded states differ"
        # Same kernel, same inputs: the results are in fact identical.
        np.testing.assert_array_equal(o_np, o_ref)
        np.testing.assert_array_equal(p_np, pool_ref)
