"""Guard bands: no call writes outside the buffers it is given.

Every output and the workspace are carved out of a larger device buffer whose
bytes before and after them hold a fill pattern (4 KiB on each side); after the
call the pattern must be intact.  The workspace is exactly moe_workspace_size
bytes.  Inputs are valid, so this is a check of the kernels' own index
arithmetic at several shapes and on every path: the single-CTA and the multi-CTA
permutation, the one-launch FFN (bf16 and E4M3 weights), the multi-launch path
with and without split-K, the stand-alone grouped FFN and combine, and the
permutation without a workspace.
"""
import ctypes

import pytest
import torch

import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GUARD = 4096
FILL = 0xA5


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    moe.load_library()


class Guarded:
    """Device buffers with fill-pattern guard bands on both sides."""

    def __init__(self):
        self.bufs = []

    def take(self, shape, dtype):
        n = 1
        for d in shape:
            n *= d
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        buf = torch.full((nbytes + 2 * GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[GUARD:GUARD + nbytes].view(dtype).view(*shape)

    def workspace(self, T, E, k, H=0, I=0):
        n = moe.moe_workspace_size(T, E, k, H, I)
        buf = torch.full((n + 2 * GUARD,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, n))
        return buf[GUARD:GUARD + n]

    def check(self, what):
        torch.cuda.synchronize()
        for i, (buf, n) in enumerate(self.bufs):
            head = buf[:GUARD]
            tail = buf[GUARD + n:]
            assert bool((head == FILL).all()), f"{what}: buffer {i} written before its start"
            assert bool((tail == FILL).all()), f"{what}: buffer {i} written past its end"


FORWARD_SHAPES = [
    ("tiny", (16, 8, 2, 256, 512)),
    ("decode_fused", (8, 128, 8, 2048, 768)),
    ("ragged_multi_launch", (100, 8, 2, 384, 640)),        # T > 64: multi-launch, split-K
    ("large_permute", (1100, 16, 4, 256, 256)),            # T*k > 4096: multi-CTA permute
    ("many_experts_fused", (40, 1024, 16, 128, 128)),
    ("nt256", (600, 4, 2, 256, 256)),                      # 256-row tiles, several per expert
]


@pytest.mark.parametrize("name,shape", FORWARD_SHAPES, ids=[s[0] for s in FORWARD_SHAPES])
def test_forward_writes_only_its_buffers(name, shape):
    T, E, k, H, I = shape
    w = wl.custom(name, T, E, k, H, I)
    d = wl.make_inputs(w, seed=21, device="cuda")
    g = Guarded()
    ws = g.workspace(T, E, k, H, I)
    out = g.take((T, H), torch.bfloat16)
    ids = g.take((T, k), torch.int32)
    wts = g.take((T, k), torch.float32)
    off = g.take((E + 1,), torch.int32)
    rows = g.take((T * k,), torch.int32)
    for _ in range(2):
        moe.moe_forward(d["x"], d["logits"], d["w13"], d["w2"], k, ws=ws, out=out, topk_ids=ids,
                        topk_weights=wts, expert_offsets=off, permuted_rows=rows)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    g.check(name)
    # the optional outputs left in the workspace
    moe.moe_forward(d["x"], d["logits"], d["w13"], d["w2"], k, ws=ws, out=out)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    g.check(name + " (outputs kept in the workspace)")


def test_forward_w8_writes_only_its_buffers():
    w = wl.WORKLOADS["decode"]
    d = wl.make_inputs(w, seed=22, device="cuda", weights=False)
    q13, s13, q2, s2 = wl.make_weights_w8(w, seed=22, device="cuda")
    g = Guarded()
    ws = g.workspace(w.T, w.E, w.k, w.H, w.I)
    out = g.take((w.T, w.H), torch.bfloat16)
    ids = g.take((w.T, w.k), torch.int32)
    wts = g.take((w.T, w.k), torch.float32)
    moe.moe_forward_w8(d["x"], d["logits"], q13, s13, q2, s2, w.k, ws=ws, out=out, topk_ids=ids,
                       topk_weights=wts)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    g.check("moe_forward_w8")


@pytest.mark.parametrize("T,E,k", [(16384, 1024, 8), (512, 8, 8), (3000, 37, 3)])
def test_route_and_permute_write_only_their_buffers(T, E, k):
    w = wl.custom("rp", T, E, k)
    logits = wl.make_logits(w, seed=23, device="cuda")
    g = Guarded()
    ids = g.take((T, k), torch.int32)
    wts = g.take((T, k), torch.float32)
    off = g.take((E + 1,), torch.int32)
    rows = g.take((T * k,), torch.int32)
    ws = g.workspace(T, E, k)
    moe.moe_route(logits, k, topk_ids=ids, topk_weights=wts)
    moe.moe_permute(ids, E, ws=ws, expert_offsets=off, permuted_rows=rows)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    g.check("moe_route + moe_permute")


def test_grouped_ffn_and_combine_write_only_their_buffers():
    T, E, k, H, I = 300, 8, 4, 256, 384
    w = wl.custom("gf", T, E, k, H, I)
    d = wl.make_inputs(w, seed=24, device="cuda")
    ids, wts = moe.moe_route(d["logits"], k)
    off, rows = moe.moe_permute(ids, E)
    g = Guarded()
    ws = g.workspace(T, E, k, H, I)
    y = g.take((T * k, H), torch.bfloat16)
    out = g.take((T, H), torch.bfloat16)
    moe.moe_grouped_ffn(d["x"], d["w13"], d["w2"], off, rows, k, ws=ws, y=y)
    moe.moe_combine(y, wts, out=out)
    assert moe.moe_device_status(ws) == moe.MOE_OK
    g.check("moe_grouped_ffn + moe_combine")


def test_permute_noalloc_writes_only_its_buffers():
    lib = moe.load_library()
    fn = lib.moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, moe.Shape, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    for T, E, k in [(8, 128, 8), (16384, 1024, 8)]:
        logits = wl.make_logits(wl.custom("na", T, E, k), seed=25, device="cuda")
        ids, _ = moe.moe_route(logits, k)
        g = Guarded()
        off = g.take((E + 1,), torch.int32)
        rows = g.take((T * k,), torch.int32)
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert fn(ctypes.c_void_p(ids.data_ptr()), moe.Shape(T, E, k, 0, 0),
                  ctypes.c_void_p(off.data_ptr()), ctypes.c_void_p(rows.data_ptr()), st) == moe.MOE_OK
        g.check(f"moe_permute_noalloc T={T} E={E}")
