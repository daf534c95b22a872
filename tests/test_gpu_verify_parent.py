"""GPU checks of the parent (not write-on-accept) verify and the fold's restore
branch, through the C ABI (page "ssm_gdn_woa.rs", gdn_wy4_fold doc: a clear
engaged word sends the fold to the kept intermediate states in hi_tables).

Against the f64 oracle (prefill tolerances): the outputs, every kept
intermediate state Hi(0..2) = the state after 1..3 rows, and the live state
left by the verify (after all four rows).  Bit-exact: a restore copies its slab
bit for bit, na = 4 leaves the verify's live state, na = 0 and a missing slab
set GDN_FLAG_ERROR and change nothing, padding sequences get zero outputs and
no state writes.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_prefill_close, f64
from linear_attention_ssm_gdn_b200 import (_lib, debug_device_errors, gdn_flag_clear, gdn_fold,
                                           gdn_verify_parent)
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(vi, slab_entries=3):
    pool = vi.pool.to(DEV).clone()
    per = pool[0].numel() * 4
    table = torch.tensor([pool.data_ptr() + int(s) * per for s in vi.slots], dtype=torch.int64,
                         device=DEV)
    slabs = torch.full((vi.batch, slab_entries) + tuple(vi.pool.shape[1:]), float("nan"),
                       device=DEV)
    sper = slabs[0, 0].numel() * 4
    hi = torch.tensor([[slabs.data_ptr() + (b * slab_entries + r) * sper
                        for r in range(slab_entries)] for b in range(vi.batch)],
                      dtype=torch.int64, device=DEV)
    d = {k: getattr(vi, k).to(DEV) for k in ("q", "k", "v", "g", "beta")}
    return pool, table, slabs, hi, d


def _oracle_after(vi, rows):
    slots = vi.slots.numpy()
    return oracle.gdn_verify_fold(f64(vi.pool)[slots], f64(vi.q), f64(vi.k), f64(vi.v),
                                  f64(vi.g), f64(vi.beta), np.full(vi.batch, rows, np.int32))


@pytest.mark.parametrize("d", [128, 64])
def test_parent_verify_states_and_outputs(d):
    vi = I.verify_inputs(12, 4, 2, 6, d, d, slots_total=16, seed=60 + d)
    pool, table, slabs, hi, dd = _setup(vi)
    o = gdn_verify_parent(table, dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], hi_tables=hi)
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    slots = vi.slots.numpy()
    o_ref, h4 = _oracle_after(vi, 4)
    assert_prefill_close(o.float().cpu().numpy(), pool.cpu().numpy()[slots], o_ref, h4,
                         f"parent d={d}: outputs, live state after 4 rows")
    for r in range(3):
        _, hr = _oracle_after(vi, r + 1)
        assert_prefill_close(np.zeros(1), slabs[:, r].cpu().numpy(), np.zeros(1), hr,
                             f"parent d={d}: Hi({r})")
    untouched = sorted(set(range(vi.pool.shape[0])) - set(slots.tolist()))
    assert torch.equal(pool[untouched].cpu(), vi.pool[untouched])


def test_fold_restores_partial_accepts_bit_for_bit():
    vi = I.verify_inputs(16, 4, 2, 4, 128, 128, slots_total=20, seed=70)
    na = torch.tensor([1, 2, 3, 4] * 4, dtype=torch.int32)
    pool, table, slabs, hi, dd = _setup(vi)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn_flag_clear(flag)
    gdn_verify_parent(table, dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], hi_tables=hi)
    torch.cuda.synchronize()
    live_after_verify = pool.cpu().clone()
    gdn_fold(table, None, na.to(DEV), dd["k"], flag, vi.H_v, hi_tables=hi)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    slots = vi.slots.numpy()
    after = pool.cpu()
    sl = slabs.cpu()
    for b in range(vi.batch):
        n = int(na[b])
        if n < 4:
            assert torch.equal(after[slots[b]], sl[b, n - 1]), f"b={b}: not the slab"
        else:
            assert torch.equal(after[slots[b]], live_after_verify[slots[b]])
    # and the restored states are the oracle's states after na rows
    ref = oracle.gdn_verify_fold(f64(vi.pool)[slots], f64(vi.q), f64(vi.k), f64(vi.v),
                                 f64(vi.g), f64(vi.beta), na.numpy())[1]
    assert_prefill_close(np.zeros(1), after.numpy()[slots], np.zeros(1), ref, "restore")


def test_fold_restore_errors_change_nothing():
    """na = 0 (the state before the verify is gone) and a NULL slab entry set
    GDN_FLAG_ERROR and skip their sequence; the others are still restored."""
    vi = I.verify_inputs(4, 4, 2, 4, 128, 128, slots_total=4, seed=71)
    pool, table, slabs, hi, dd = _setup(vi)
    hi[2, 1] = 0  # sequence 2 keeps no Hi(1)
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    gdn_flag_clear(flag)
    gdn_verify_parent(table, dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], hi_tables=hi)
    torch.cuda.synchronize()
    live = pool.cpu().clone()
    na = torch.tensor([0, 2, 2, 5], dtype=torch.int32, device=DEV)
    gdn_fold(table, None, na, dd["k"], flag, vi.H_v, hi_tables=hi)
    torch.cuda.synchronize()
    assert int(flag.item()) == _lib.GDN_FLAG_ERROR
    slots = vi.slots.numpy()
    after = pool.cpu()
    for b in (0, 2, 3):
        assert torch.equal(after[slots[b]], live[slots[b]])
    assert torch.equal(after[slots[1]], slabs[1, 1].cpu())


def test_parent_padding_and_no_slabs():
    """A NULL table entry is a padding sequence (zero outputs, nothing
    written); without hi_tables the verify still writes the live state; a
    restore copies whatever its slab holds (here never written: NaN)."""
    vi = I.verify_inputs(3, 4, 1, 2, 64, 64, slots_total=3, seed=72)
    pool, table, slabs, hi, dd = _setup(vi)
    table[1] = 0
    o = torch.full((12, vi.H_v, 64), 3.0, dtype=torch.bfloat16, device=DEV)
    gdn_verify_parent(table, dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], o=o)
    torch.cuda.synchronize()
    assert torch.all(o[4:8] == 0)
    assert torch.equal(pool[vi.slots[1]].cpu(), vi.pool[vi.slots[1]])
    assert torch.isnan(slabs).all()  # no slab was given, none written
    slots = vi.slots.numpy()
    _, h4 = _oracle_after(vi, 4)
    for b in (0, 2):
        assert_prefill_close(np.zeros(1), pool.cpu().numpy()[slots[b]][None], np.zeros(1),
                             h4[b][None], f"live b={b}")
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    live = pool.clone()
    # engaged word clear, slabs never written (still NaN): a restore copies them
    gdn_fold(table, None, torch.tensor([1, 1, 1], dtype=torch.int32, device=DEV), dd["k"], flag,
             vi.H_v, hi_tables=hi)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert torch.isnan(pool[vi.slots[0]]).all() and torch.equal(pool[vi.slots[1]], live[vi.slots[1]])
