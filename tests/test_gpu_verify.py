"""GPU checks of gdn_flag_clear / gdn_verify_woa / gdn_fold (through the C ABI).

Outputs and folded states against the f64 oracle (5e-3 / 2e-2); the
bit-exact facts: na = 0 leaves a state bit-identical, verify writes no state,
pool slots outside the table are untouched, swapping table entries swaps the
results exactly, and a clear engaged word makes the fold a no-op.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import assert_prefill_close, f64
from linear_attention_ssm_gdn_b200 import _lib
from linear_attention_ssm_gdn_b200 import (debug_device_errors, gdn_flag_clear, gdn_fold,
                                           gdn_verify_woa)
from linear_attention_ssm_gdn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _setup(vi: I.VerifyInputs):
    pool = vi.pool.to(DEV).clone()
    per_slot = pool[0].numel() * 4
    table = torch.tensor([pool.data_ptr() + int(s) * per_slot for s in vi.slots],
                         dtype=torch.int64, device=DEV)
    dev = {k: getattr(vi, k).to(DEV) for k in ("q", "k", "v", "g", "beta", "na")}
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    return pool, table, dev, flag


def _verify_fold(vi, na=None, clear=True, fold=True):
    pool, table, d, flag = _setup(vi)
    if clear:
        gdn_flag_clear(flag)
    o, stash = gdn_verify_woa(table, d["q"], d["k"], d["v"], d["g"], d["beta"], flag)
    torch.cuda.synchronize()
    pool_after_verify = pool.cpu().clone()
    na_t = d["na"] if na is None else torch.as_tensor(na, dtype=torch.int32, device=DEV)
    if fold:
        gdn_fold(table, stash, na_t, d["k"], flag, vi.H_v)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), pool.cpu(), pool_after_verify, int(flag.item())


def test_verify_fold_full_size_against_oracle():
    vi = I.workload(4).verify
    o, pool, pool_v, flag = _verify_fold(vi)
    assert debug_device_errors() == [0, 0, 0, 0]
    assert flag == 1
    assert torch.equal(pool_v, vi.pool)  # verify wrote no state
    slots = vi.slots.numpy()
    hs = f64(vi.pool)[slots]
    o_ref, h_ref = oracle.gdn_verify_fold(hs, f64(vi.q), f64(vi.k), f64(vi.v), f64(vi.g),
                                          f64(vi.beta), vi.na.numpy())
    assert_prefill_close(o, pool.numpy()[slots], o_ref, h_ref, "verify/fold")
    na = vi.na.numpy()
    for b in np.nonzero(na == 0)[0]:  # na = 0: bit-identical
        assert torch.equal(pool[slots[b]], vi.pool[slots[b]])
    untouched = sorted(set(range(vi.pool.shape[0])) - set(slots.tolist()))
    assert torch.equal(pool[untouched], vi.pool[untouched])


def test_fold_all_accepted_equals_four_steps():
    vi = I.verify_inputs(8, 4, 2, 4, 128, 128, slots_total=12, seed=40)
    _, pool, _, _ = _verify_fold(vi, na=[4] * 8)
    slots = vi.slots.numpy()
    for b in range(8):
        sl = slice(4 * b, 4 * b + 4)
        _, h_ref = oracle.gdn_token(f64(vi.q)[sl], f64(vi.k)[sl], f64(vi.v)[sl], f64(vi.g)[sl],
                                    f64(vi.beta)[sl], [0, 4], f64(vi.pool)[slots[b]][None])
        assert_prefill_close(np.zeros(1), pool.numpy()[slots[b]][None], np.zeros(1), h_ref,
                             f"b={b}")


def test_fold_with_flag_clear_is_a_no_op():
    vi = I.verify_inputs(6, 4, 2, 4, 128, 128, slots_total=8, seed=41)
    pool, table, d, flag = _setup(vi)
    _, stash = gdn_verify_woa(table, d["q"], d["k"], d["v"], d["g"], d["beta"], flag)
    gdn_flag_clear(flag)  # verdict arrives after a clear: nothing may change
    gdn_fold(table, stash, torch.full((6,), 4, dtype=torch.int32, device=DEV), d["k"], flag,
             vi.H_v)
    torch.cuda.synchronize()
    assert torch.equal(pool.cpu(), vi.pool)


def test_fold_after_a_failed_verify_changes_no_state():
    """A verify CTA whose bounded wait ran out ORs GDN_FLAG_ERROR |
    GDN_FLAG_STASH_BAD into the engaged word (its stash is incomplete).  The
    bits are planted on the host here, between a normal verify and the fold:
    the fold must then leave every state bit-identical, whatever na says."""
    vi = I.verify_inputs(6, 4, 2, 4, 128, 128, slots_total=8, seed=47)
    pool, table, d, flag = _setup(vi)
    gdn_flag_clear(flag)
    _, stash = gdn_verify_woa(table, d["q"], d["k"], d["v"], d["g"], d["beta"], flag)
    flag.bitwise_or_(_lib.GDN_FLAG_ERROR | _lib.GDN_FLAG_STASH_BAD)
    gdn_fold(table, stash, torch.full((6,), 4, dtype=torch.int32, device=DEV), d["k"], flag,
             vi.H_v)
    torch.cuda.synchronize()
    assert int(flag.item()) == 7
    assert torch.equal(pool.cpu(), vi.pool)


def test_fold_bad_na_sets_error_bit_and_skips():
    vi = I.verify_inputs(4, 4, 2, 4, 128, 128, slots_total=4, seed=42)
    _, pool, _, flag = _verify_fold(vi, na=[5, -1, 0, 2])
    assert flag & 2 and flag & 1
    slots = vi.slots.numpy()
    for b in (0, 1, 2):
        assert torch.equal(pool[slots[b]], vi.pool[slots[b]])
    assert not torch.equal(pool[slots[3]], vi.pool[slots[3]])


def test_table_routing_is_exact():
    """Swapping two table entries swaps the two results bit for bit."""
    vi = I.verify_inputs(4, 4, 2, 4, 128, 128, slots_total=6, seed=43)
    na = [4, 4, 4, 4]
    _, pool1, _, _ = _verify_fold(vi, na=na)
    vi2 = I.verify_inputs(4, 4, 2, 4, 128, 128, slots_total=6, seed=43)
    s = vi2.slots.clone()
    vi2.slots[0], vi2.slots[1] = s[1], s[0]
    # swap the rows of sequences 0 and 1 too, so each state sees the same rows
    for name in ("q", "k", "v", "g", "beta"):
        t = getattr(vi2, name).clone()
        t[0:4], t[4:8] = getattr(vi2, name)[4:8], getattr(vi2, name)[0:4]
        setattr(vi2, name, t)
    _, pool2, _, _ = _verify_fold(vi2, na=na)
    assert torch.equal(pool1, pool2)


def test_null_table_entry_is_padding():
    vi = I.verify_inputs(3, 4, 2, 4, 128, 128, slots_total=3, seed=44)
    pool, table, d, flag = _setup(vi)
    table[1] = 0
    gdn_flag_clear(flag)
    o = torch.full((12, vi.H_v, 128), 3.0, dtype=torch.bfloat16, device=DEV)
    _, stash = gdn_verify_woa(table, d["q"], d["k"], d["v"], d["g"], d["beta"], flag, o=o)
    gdn_fold(table, stash, torch.full((3,), 4, dtype=torch.int32, device=DEV), d["k"], flag,
             vi.H_v)
    torch.cuda.synchronize()
    assert torch.all(o[4:8] == 0)
    assert torch.equal(pool[vi.slots[1]].cpu(), vi.pool[vi.slots[1]])


def test_d64_heads():
    vi = I.verify_inputs(5, 4, 1, 3, 64, 64, slots_total=7, seed=45)
    o, pool, _, _ = _verify_fold(vi)
    slots = vi.slots.numpy()
    o_ref, h_ref = oracle.gdn_verify_fold(f64(vi.pool)[slots], f64(vi.q), f64(vi.k), f64(vi.v),
                                          f64(vi.g), f64(vi.beta), vi.na.numpy())
    assert_prefill_close(o, pool.numpy()[slots], o_ref, h_ref, "d=64")


@pytest.mark.parametrize("batch,H_k,H_v,d", [(150, 2, 4, 128), (240, 2, 6, 64)])
def test_many_items_per_cta_with_padding(batch, H_k, H_v, d):
    """More (sequence, v-head) items than SMs, every third sequence a padding
    entry: each persistent CTA walks several items, and its half-state ring
    (4 slots at d = 128, 16 at d = 64) wraps across padding items, which
    take no slot.  Outputs and folded states of the present sequences match
    the oracle; padding rows are zero and their states bit-identical."""
    vi = I.verify_inputs(batch, 4, H_k, H_v, d, d, slots_total=batch + 3, seed=46 + d)
    pool, table, dd, flag = _setup(vi)
    present = np.ones(batch, dtype=np.int32)
    present[::3] = 0
    for b in np.nonzero(present == 0)[0]:
        table[int(b)] = 0
    gdn_flag_clear(flag)
    o, stash = gdn_verify_woa(table, dd["q"], dd["k"], dd["v"], dd["g"], dd["beta"], flag)
    gdn_fold(table, stash, dd["na"], dd["k"], flag, vi.H_v)
    torch.cuda.synchronize()
    assert debug_device_errors() == [0, 0, 0, 0]
    slots = vi.slots.numpy()
    o_ref, h_ref = oracle.gdn_verify_fold(f64(vi.pool)[slots], f64(vi.q), f64(vi.k), f64(vi.v),
                                          f64(vi.g), f64(vi.beta), vi.na.numpy(), present=present)
    o_np = o.float().cpu().numpy()
    pool_after = pool.cpu()
    assert_prefill_close(o_np, pool_after.numpy()[slots], o_ref, h_ref, f"padded d={d}")
    for b in np.nonzero(present == 0)[0]:
        assert np.all(o_np[4 * b:4 * b + 4] == 0)
        assert torch.equal(pool_after[slots[b]], vi.pool[slots[b]])
