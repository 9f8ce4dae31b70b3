"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (no workspace argument; its scratch is a fixed array inside the library).

Checked through the C ABI against moe_permute, the entry point that takes a
workspace: the results must be bit-identical, on two calls in a row (the second
call must not be disturbed by what the first left in the shared array).  This
file is collected last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.  (Its
rejection of sizes beyond the scratch is checked on the host, without a device,
in test_boundary.py.)
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_logits_b200 as moe

MAX_ROWS = 1 << 20


def _lib():
    from mixture_experts_layer_logits_b200 import build

    build.build()
    lib = moe.load_library()
    fn = lib.moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, moe.Shape, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return lib


def _ids(T, E, k, seed, hot=False):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    if hot:
        logits[:, 0] += 4.0
    return torch.topk(logits, k, dim=1).indices.to(torch.int32).contiguous()


def _noalloc(lib, ids, E):
    T, k = ids.shape
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    rows = torch.full((T * k,), -7, dtype=torch.int32, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.moe_permute_noalloc(ctypes.c_void_p(ids.data_ptr()), moe.Shape(T, E, k, 0, 0),
                                 ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(rows.data_ptr()),
                                 st)
    assert rc == moe.MOE_OK, lib.moe_status_string(rc).decode()
    return off, rows


def _with_workspace(ids, E):
    T, k = ids.shape
    ws = moe.workspace(T, E, k)
    return moe.moe_permute(ids, E, ws=ws)


# the last case fills the scratch to its limit: T*k = 2^20 rows, 512 chunks of
# counts at E = 1024, right below the tile list
CASES = [(8, 128, 8, False), (16384, 1024, 8, False), (5000, 37, 3, True), (512, 8, 8, False),
         (70000, 256, 8, True), (MAX_ROWS // 8, 1024, 8, True)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_permute_on_consecutive_calls():
    lib = _lib()
    for i, (T, E, k, hot) in enumerate(CASES):
        a = _ids(T, E, k, seed=100 + i, hot=hot).cuda()
        b = _ids(T, E, k, seed=200 + i, hot=not hot).cuda()
        got_a = _noalloc(lib, a, E)          # first call
        got_b = _noalloc(lib, b, E)          # second call, right after, same shared scratch
        want_a = _with_workspace(a, E)
        want_b = _with_workspace(b, E)
        torch.cuda.synchronize()
        for got, want in ((got_a, want_a), (got_b, want_b)):
            np.testing.assert_array_equal(got[0].cpu().numpy(), want[0].cpu().numpy())
            np.testing.assert_array_equal(got[1].cpu().numpy(), want[1].cpu().numpy())
