"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory at call time (its scratch is an array built into the
library).  Called through the C ABI and compared, bit for bit, with the
float64 oracle's permutation and with the workspace-based moe_permute, on
calls made back to back; the second call has a different shape, so stale
scratch from the first would show.  Batches of up to 8192 slots are
permuted inside one block without any scratch, so the main calls use 32,768
and 16,384 slots (through the scratch array), and one more call of 2,048
slots covers the one-block path."""
import ctypes

import numpy as np
import pytest

import oracle
import routed_expert_ffn_prefix_b200 as moe
from routed_expert_ffn_prefix_b200 import build as moe_build

pytestmark = pytest.mark.gpu


def _noalloc():
    moe_build.build()
    fn = moe.lib().moe_permute_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [P, I, I, I, P, P, P, P, P]
    fn.restype = I
    return fn


def _ids(rng, T, E, k):
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)


def _call(fn, ids, T, E, k):
    import torch
    got = (torch.full((E,), -1, dtype=torch.int32, device="cuda"),
           torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
           torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
           torch.full((T, k), -1, dtype=torch.int32, device="cuda"))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = fn(ctypes.c_void_p(ids.data_ptr()), T, E, k, *[ctypes.c_void_p(g.data_ptr()) for g in got], stream)
    assert st == 0, moe.STATUS.get(st, st)
    torch.cuda.synchronize()
    return [g.cpu().numpy() for g in got]


def test_noalloc_permute_matches_oracle_and_workspace_permute_twice():
    import torch
    fn = _noalloc()
    rng = np.random.default_rng(11)
    for T, E, k in [(4096, 256, 8), (2048, 512, 8), (256, 64, 8)]:
        ids_h = _ids(rng, T, E, k)
        ids = torch.from_numpy(ids_h).cuda()
        got = _call(fn, ids, T, E, k)
        counts, offsets, sids, inv = oracle.permute(ids_h, E)
        np.testing.assert_array_equal(got[0], counts)
        np.testing.assert_array_equal(got[1], offsets)
        np.testing.assert_array_equal(got[2], sids)
        np.testing.assert_array_equal(got[3], inv)
        ws = moe.alloc_workspace(T, 256, E, 128, k)
        want = moe.permute(ids, E, ws)
        assert moe.device_status(ws) == 0
        for g, w in zip(got, want):
            np.testing.assert_array_equal(g, w.cpu().numpy())


@pytest.mark.parametrize("T,E,k", [(4096, 256, 8), (512, 64, 4)])
def test_noalloc_permute_skips_out_of_range_ids(T, E, k):
    """Ids of -1 and E are skipped: counts and offsets cover only the valid
    slots, the valid slots keep the order the oracle gives them, and the
    skipped slots' inv_perm entries are left as the caller's buffer held
    them (-1 here)."""
    import torch
    fn = _noalloc()
    rng = np.random.default_rng(5)
    ids_h = _ids(rng, T, E, k)
    bad = rng.choice(T * k, size=37, replace=False)
    flat = ids_h.reshape(-1)
    flat[bad[::2]] = -1
    flat[bad[1::2]] = E
    got = _call(fn, torch.from_numpy(ids_h).cuda(), T, E, k)
    valid = (flat >= 0) & (flat < E)
    assert int(got[0].sum()) == T * k - bad.size
    assert got[1][E] == T * k - bad.size
    # The oracle on the valid slots alone: rows are expert-major, then slot order.
    slots = np.nonzero(valid)[0]
    order = slots[np.lexsort((slots, flat[slots]))]
    np.testing.assert_array_equal(got[0], np.bincount(flat[slots], minlength=E))
    np.testing.assert_array_equal(got[2][:order.size], order // k)
    inv = got[3].reshape(-1)
    np.testing.assert_array_equal(inv[order], np.arange(order.size))
    assert np.all(inv[~valid] == -1)


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    fn = _noalloc()
    F = ctypes.c_void_p(0x100000)  # never used: the size check fails first
    assert fn(F, 20000, 512, 10, F, F, F, F, None) == 3   # T*k = 200000 > 131072: MOE_ERR_WORKSPACE
    assert fn(F, 4, 2048, 2, F, F, F, F, None) == 1        # E > 1024: MOE_ERR_INVALID_ARG, as moe_permute
