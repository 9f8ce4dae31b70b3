"""The debug build (libmoe_debug.so, compiled with MOE_DEBUG).

Its kernels check the indices they read from their inputs -- expert ids given to
moe_permute, expert offsets and permuted rows given to moe_grouped_ffn -- and on
a violation record MOE_ERR_DEVICE_BOUNDS in the workspace's error word and skip
(or redirect to index 0) the access instead of making it.

1. On valid inputs the debug build returns exactly what the release build
   returns (same kernels, the checks only compiled in) and reports no error.
2. Out-of-range ids, offsets and rows make it report MOE_ERR_DEVICE_BOUNDS,
   nothing outside the given buffers is written (guard bands), and the context
   stays usable: a valid call right after returns the right result.

The release library is already loaded in the test process, so the debug build
runs in a child process (MOE_LIBRARY=debug) that saves its results to a file.
"""
import os
import subprocess
import sys

import pytest
import torch

import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    moe.load_library()


FORWARD_SHAPES = [(16, 8, 2, 256, 512), (8, 128, 8, 2048, 768), (100, 8, 2, 384, 640),
                  (1100, 16, 4, 256, 256), (600, 4, 2, 256, 256)]
ROUTING_SHAPES = [(16384, 1024, 8), (512, 8, 8)]

CHILD = r'''
import os, sys, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))
import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl
from test_gpu_debug import FORWARD_SHAPES, ROUTING_SHAPES, run_valid, run_invalid
assert moe.library_path == moe.debug_library_path
moe.load_library()
torch.save({"valid": run_valid(), "invalid": run_invalid()}, sys.argv[1])
'''


def run_valid():
    """Outputs of a few calls on valid inputs, with the status after each."""
    res = {}
    for T, E, k, H, I in FORWARD_SHAPES:
        w = wl.custom("d", T, E, k, H, I)
        d = wl.make_inputs(w, seed=31, device="cuda")
        ws = moe.workspace(T, E, k, H, I)
        ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
        out = moe.moe_forward(d["x"], d["logits"], d["w13"], d["w2"], k, ws=ws, topk_ids=ids)
        res[("forward", T, E, k, H, I)] = (out.cpu(), ids.cpu(), moe.moe_device_status(ws))
    for T, E, k in ROUTING_SHAPES:
        logits = wl.make_logits(wl.custom("r", T, E, k), seed=32, device="cuda")
        ws = moe.workspace(T, E, k)
        ids, wts = moe.moe_route(logits, k)
        off, rows = moe.moe_permute(ids, E, ws=ws)
        res[("routing", T, E, k)] = (ids.cpu(), wts.cpu(), off.cpu(), rows.cpu(),
                                     moe.moe_device_status(ws))
    return res


GUARD = 4096


def _guarded(n, dtype):
    es = torch.tensor([], dtype=dtype).element_size()
    buf = torch.full((n * es + 2 * GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    return buf, buf[GUARD:GUARD + n * es].view(dtype)


def _intact(buf):
    torch.cuda.synchronize()
    return bool((buf[:GUARD] == 0xA5).all()) and bool((buf[-GUARD:] == 0xA5).all())


def run_invalid():
    """Out-of-range inputs: (status, guard bands intact, the valid call right after correct)."""
    res = {}
    # expert ids outside [0, E): the single-CTA (T*k <= 4096) and the multi-CTA permutation
    for T, E, k in [(64, 32, 4), (2000, 64, 4)]:
        logits = wl.make_logits(wl.custom("p", T, E, k), seed=33, device="cuda")
        ids, _ = moe.moe_route(logits, k)
        good_off, good_rows = moe.moe_permute(ids, E)
        bad = ids.clone()
        bad[1, 0] = E
        bad[T - 1, k - 1] = -1
        ws = moe.workspace(T, E, k)
        ob, off = _guarded(E + 1, torch.int32)
        rb, rows = _guarded(T * k, torch.int32)
        moe.moe_permute(bad, E, ws=ws, expert_offsets=off, permuted_rows=rows)
        st = moe.moe_device_status(ws)
        guards = _intact(ob) and _intact(rb)
        moe.moe_permute(ids, E, ws=ws, expert_offsets=off, permuted_rows=rows)
        after = (moe.moe_device_status(ws) == moe.MOE_OK and torch.equal(off, good_off)
                 and torch.equal(rows, good_rows))
        res[("permute_ids", T, E, k)] = (st, guards, after)
    # moe_grouped_ffn: a permuted row past T*k, then expert offsets past T*k
    T, E, k, H, I = 300, 8, 4, 256, 384
    w = wl.custom("g", T, E, k, H, I)
    d = wl.make_inputs(w, seed=34, device="cuda")
    ids, wts = moe.moe_route(d["logits"], k)
    off, rows = moe.moe_permute(ids, E)
    good_y = moe.moe_grouped_ffn(d["x"], d["w13"], d["w2"], off, rows, k)
    for what in ("row", "offsets"):
        r2, o2 = rows.clone(), off.clone()
        if what == "row":
            r2[5] = T * k + 7
        else:
            o2[E] = T * k + 100
            o2[3] = o2[2] - 1
        ws = moe.workspace(T, E, k, H, I)
        yb, y = _guarded(T * k * H, torch.bfloat16)
        y = y.view(T * k, H)
        moe.moe_grouped_ffn(d["x"], d["w13"], d["w2"], o2, r2, k, ws=ws, y=y)
        st = moe.moe_device_status(ws)
        guards = _intact(yb)
        moe.moe_grouped_ffn(d["x"], d["w13"], d["w2"], off, rows, k, ws=ws, y=y)
        after = moe.moe_device_status(ws) == moe.MOE_OK and torch.equal(y, good_y)
        res[("grouped_ffn", what)] = (st, guards, after)
    return res


def test_debug_build_matches_release_and_catches_bad_indices(tmp_path):
    path = tmp_path / "debug.pt"
    script = tmp_path / "child.py"
    script.write_text(f"ROOT = {ROOT!r}\n" + CHILD)
    env = dict(os.environ, MOE_LIBRARY="debug")
    subprocess.run([sys.executable, str(script), str(path)], env=env, check=True, timeout=900)
    got = torch.load(path)
    # 1. valid inputs: identical to the release build, no error reported
    want = run_valid()
    for key, ref in want.items():
        dbg = got["valid"][key]
        assert dbg[-1] == moe.MOE_OK and ref[-1] == moe.MOE_OK, key
        for a, b in zip(dbg[:-1], ref[:-1]):
            assert torch.equal(a, b), key
    # 2. out-of-range inputs: reported, contained, recovered from
    for key, (st, guards, after) in got["invalid"].items():
        assert st == moe.MOE_ERR_DEVICE_BOUNDS, (key, st)
        assert guards, f"{key}: a guard band was overwritten"
        assert after, f"{key}: the valid call after it went wrong"
