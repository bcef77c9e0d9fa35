"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory at call time (its scratch is an array built into the
library).  Called through the C ABI and compared, bit for bit, with the
workspace-based moe_permute on two calls in a row; the second call has a
different shape so stale scratch from the first would show.  Batches of up
to 8192 slots are permuted inside one block without any scratch, so the
calls use 32,768 and 16,384 slots, which go through the scratch array."""
import ctypes

import numpy as np
import pytest

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


def test_noalloc_permute_matches_workspace_permute_twice():
    import torch
    fn = _noalloc()
    rng = np.random.default_rng(11)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for T, E, k in [(4096, 256, 8), (2048, 512, 8)]:
        ids = torch.from_numpy(_ids(rng, T, E, k)).cuda()
        ws = moe.alloc_workspace(T, 256, E, 128, k)
        want = moe.permute(ids, E, ws)
        assert moe.device_status(ws) == 0
        got = (torch.full((E,), -1, dtype=torch.int32, device="cuda"),
               torch.full((E + 1,), -1, dtype=torch.int32, device="cuda"),
               torch.full((T * k,), -1, dtype=torch.int32, device="cuda"),
               torch.full((T, k), -1, dtype=torch.int32, device="cuda"))
        st = fn(ctypes.c_void_p(ids.data_ptr()), T, E, k, *[ctypes.c_void_p(g.data_ptr()) for g in got], stream)
        assert st == 0, moe.STATUS.get(st, st)
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            assert torch.equal(g, w)


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    fn = _noalloc()
    F = ctypes.c_void_p(0x100000)  # never used: the size check fails first
    assert fn(F, 20000, 512, 10, F, F, F, F, None) == 3   # T*k = 200000 > 131072
    assert fn(F, 4, 2048, 2, F, F, F, F, None) == 3        # E > 1024
