"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle on a B200.

Every input is seeded and synthetic (mixture_experts_layer_logits_b200.workloads);
the oracle receives host copies of the exact tensors the kernels consumed.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl

from parity import (assert_out_close, assert_routing_equal, expert_weights_for, host_bits,
                    host_f32, library_tile_rows, tile_boundary_tokens)

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    moe.load_library()


def inputs(w, seed=0):
    return wl.make_inputs(w, seed=seed, device="cuda")


# ------------------------------------------------------------------ routing

ROUTE_CASES = ["tiny", "decode", "skewed_decode", "routing_stress", "prefill"]


@pytest.mark.parametrize("name", ROUTE_CASES)
def test_route_matches_oracle(name):
    w = wl.WORKLOADS[name]
    logits = wl.make_logits(w, device="cuda")
    ids, wts = moe.moe_route(logits, w.k)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.route(host_f32(logits), w.k)
    assert_routing_equal(ids, wts, ref_ids, ref_w)


def adversarial_logits(T, E, seed):
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(T, E, generator=g)
    pool = torch.tensor([0.0, -0.0, 1.0, -1.0, 2.5, float("-inf"), 7.0])
    mask = torch.rand(T, E, generator=g) < 0.5
    a[mask] = pool[torch.randint(0, len(pool), (int(mask.sum()),), generator=g)]
    a[0] = 0.0                                 # all equal
    a[1] = -0.0
    a[1, ::2] = 0.0                            # alternating signed zeros
    if T > 2:
        a[2] = float("-inf")
        a[2, E // 2] = 1.0                     # one finite, the rest -inf
    if T > 3:
        a[3] = torch.arange(E, dtype=torch.float32) % 3   # ties at the k-th/(k+1)-th boundary
    # a row whose logits are all -inf has NaN weights: outside the contract
    dead = torch.isinf(a).all(dim=1)
    a[dead, 0] = 0.5
    return a.contiguous()


@pytest.mark.parametrize("E,k", [(8, 2), (8, 8), (128, 8), (256, 8), (1024, 8), (1000, 16),
                                 (1, 1), (33, 5), (64, 16), (300, 1)])
def test_route_adversarial_ties(E, k):
    logits = adversarial_logits(64, E, seed=E * 31 + k)
    ids, wts = moe.moe_route(logits.cuda(), k)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.route(logits.numpy(), k)
    assert_routing_equal(ids, wts, ref_ids, ref_w)


@pytest.mark.parametrize("T,E,k", [(63, 1024, 16), (63, 1000, 8), (7, 512, 8), (33, 300, 16),
                                   (5, 260, 1), (129, 772, 4)])
def test_route_many_experts_odd_counts(T, E, k):
    """256 < E <= 1024 (the streaming router: 16 or 32 values per lane, rows
    staged in shared memory) with token counts that leave the last CTA partly
    idle, experts that do not fill the last float4 slots, and ties that push
    tokens onto the exact path."""
    logits = adversarial_logits(T, E, seed=T * 7 + E + k)
    ids, wts = moe.moe_route(logits.cuda(), k)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.route(logits.numpy(), k)
    assert_routing_equal(ids, wts, ref_ids, ref_w)


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("T,E,k,hot", [(16, 8, 2, False), (8, 128, 8, False), (64, 256, 8, True),
                                       (512, 8, 8, False),      # R = 4096: single-CTA path
                                       (513, 8, 8, False),      # R = 4104: multi-CTA path
                                       (16384, 1024, 8, False), (8192, 128, 8, True),
                                       (3000, 1, 1, False), (5000, 37, 3, True),
                                       # > 148 x 8192 rows: chunks too large to stage in
                                       # shared memory, ids read from global memory twice
                                       (200000, 64, 8, True)])
def test_permute_matches_oracle(T, E, k, hot):
    g = torch.Generator().manual_seed(T + E)
    logits = torch.randn(T, E, generator=g)
    if hot:
        logits[:, 0] += 4.0                    # one expert takes (almost) every token
        if E > 2:
            logits[:, E - 1] -= 100.0          # and one takes none
    ref_ids, _ = oracle.route(logits.numpy(), k)
    ref_off, ref_rows = oracle.permute(ref_ids, E)
    ids = torch.from_numpy(ref_ids).cuda()
    off, rows = moe.moe_permute(ids, E)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)


def test_routing_stress_full_route_and_permute():
    w = wl.WORKLOADS["routing_stress"]
    logits = wl.make_logits(w, device="cuda")
    ids, wts = moe.moe_route(logits, w.k)
    off, rows = moe.moe_permute(ids, w.E)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.route(host_f32(logits), w.k)
    ref_off, ref_rows = oracle.permute(ref_ids, w.E)
    assert_routing_equal(ids, wts, ref_ids, ref_w)
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)


# ------------------------------------------------------------------ whole layer

def run_forward(w, d):
    T, E, k = w.T, w.E, w.k
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, k, dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rows = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = moe.workspace(T, E, k, w.H, w.I)
    out = moe.moe_forward(d["x"], d["logits"], d["w13"], d["w2"], k, ws=ws, topk_ids=ids,
                          topk_weights=wts, expert_offsets=off, permuted_rows=rows)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == moe.MOE_OK
    return out, ids, wts, off, rows


def check_full(w, d):
    out, ids, wts, off, rows = run_forward(w, d)
    ref = oracle.forward(host_bits(d["x"]), host_f32(d["logits"]), host_bits(d["w13"]),
                         host_bits(d["w2"]), w.k)
    assert_routing_equal(ids, wts, ref["topk_ids"], ref["topk_weights"])
    np.testing.assert_array_equal(off.cpu().numpy(), ref["expert_offsets"])
    np.testing.assert_array_equal(rows.cpu().numpy(), ref["permuted_rows"])
    return assert_out_close(out, ref["out"])


@pytest.mark.parametrize("name", ["tiny", "decode"])
def test_forward_full_configs(name):
    w = wl.WORKLOADS[name]
    check_full(w, inputs(w))


def check_tokens(w, d, pick):
    """Routing and permutation in full; the layer output of the tokens that
    pick(ref_offsets, ref_rows) lists against the oracle's forward_tokens (a
    token's output depends only on its own row), with host copies of only the
    experts those tokens select."""
    out, ids, wts, off, rows = run_forward(w, d)
    ref_ids, ref_w = oracle.route(host_f32(d["logits"]), w.k)
    assert_routing_equal(ids, wts, ref_ids, ref_w)
    ref_off, ref_rows = oracle.permute(ref_ids, w.E)
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    toks = pick(ref_off, ref_rows)
    w13s, w2s = expert_weights_for(toks, ref_ids, d["w13"], d["w2"])
    ref = oracle.forward_tokens(host_bits(d["x"]), host_f32(d["logits"]), w13s, w2s, w.k, toks,
                                w.I)
    return assert_out_close(out[toks], ref, what=f"out[{len(toks)} of {w.T} tokens]")


def test_forward_skewed_decode_all_tokens():
    """The skewed-decode layer (T=64, E=256, k=8, H=7168, I=2048, Zipf-hot experts)
    against the oracle on every token."""
    w = wl.WORKLOADS["skewed_decode"]
    d = inputs(w)
    check_tokens(w, d, lambda off, rows: list(range(w.T)))
    del d
    torch.cuda.empty_cache()


def test_forward_prefill_every_tile():
    """The prefill layer (T=8192, E=128, k=8, H=4096, I=1536) against the oracle on
    every token whose row is the first or the last row of a 256-row tile of an
    expert's segment: every (expert, tile) of both grouped GEMMs, every ragged
    tail and every segment boundary holds a checked row, and the other rows of
    those tokens land anywhere inside other tiles."""
    w = wl.WORKLOADS["prefill"]
    d = inputs(w)
    nt = library_tile_rows(w.T)
    assert nt == 256

    def pick(off, rows):
        toks = tile_boundary_tokens(off, rows, w.k, nt)
        checked = np.zeros(w.T * w.k, bool)
        for t in toks:
            checked[t * w.k:(t + 1) * w.k] = True
        # every tile of every expert holds at least one checked row
        for e in range(w.E):
            for s in range(int(off[e]), int(off[e + 1]), nt):
                assert checked[rows[s:min(s + nt, int(off[e + 1]))]].any(), (e, s)
        return toks

    check_tokens(w, d, pick)
    del d
    torch.cuda.empty_cache()


EDGE = [
    # name, T, E, k, H, I, zipf
    ("one_token_one_expert", 1, 1, 1, 128, 128, 0.0),
    ("k_equals_E", 5, 8, 8, 256, 128, 0.0),
    ("ragged_tiles", 37, 6, 3, 384, 640, 0.0),          # N tail, several 128-row blocks
    ("nt32", 17, 16, 4, 256, 256, 0.0),
    ("nt128", 100, 8, 2, 128, 384, 0.0),
    ("nt256_multi_tile", 300, 4, 2, 256, 256, 0.0),      # >256 rows per expert
    ("hot_expert_zipf", 200, 64, 4, 512, 256, 2.5),      # most experts empty
    ("large_permute_path", 1100, 16, 4, 128, 128, 0.0),  # R > 4096 -> multi-CTA permute
    ("many_experts", 40, 1024, 16, 128, 128, 0.0),
]


@pytest.mark.parametrize("name,T,E,k,H,I,zipf", EDGE, ids=[e[0] for e in EDGE])
def test_forward_edge_shapes(name, T, E, k, H, I, zipf):
    w = wl.custom(name, T, E, k, H, I, zipf_s=zipf)
    check_full(w, inputs(w, seed=3))


def test_grouped_ffn_and_combine_entry_points():
    w = wl.custom("standalone", 24, 16, 4, 256, 384)
    d = inputs(w, seed=5)
    ref_ids, ref_w = oracle.route(host_f32(d["logits"]), w.k)
    ref_off, ref_rows = oracle.permute(ref_ids, w.E)
    y = moe.moe_grouped_ffn(d["x"], d["w13"], d["w2"], torch.from_numpy(ref_off).cuda(),
                            torch.from_numpy(ref_rows).cuda(), w.k)
    torch.cuda.synchronize()
    ref_y = oracle.ffn(host_bits(d["x"]), host_bits(d["w13"]), host_bits(d["w2"]), ref_off,
                       ref_rows, w.k)
    assert_out_close(y, ref_y, what="y")
    wts = torch.from_numpy(ref_w).cuda()
    out = moe.moe_combine(y, wts)
    torch.cuda.synchronize()
    # combine alone: oracle combine of the GPU's own y (same bf16 values)
    ref_out = oracle.combine(y.float().cpu().double().numpy(), ref_w)
    got = out.float().cpu().double().numpy()
    # fp32 fixed-order sum of k terms, then one bf16 rounding
    np.testing.assert_allclose(got, ref_out, rtol=2 ** -8, atol=1e-6)


def test_forward_is_deterministic():
    w = wl.WORKLOADS["decode"]
    d = inputs(w, seed=7)
    a = run_forward(w, d)[0].clone()
    b = run_forward(w, d)[0].clone()
    assert torch.equal(a, b)


def test_forward_without_pdl_is_identical(tmp_path):
    script = tmp_path / "nopdl.py"
    script.write_text(
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import mixture_experts_layer_logits_b200 as moe\n"
        "from mixture_experts_layer_logits_b200 import workloads as wl\n"
        "w = wl.WORKLOADS['decode']\n"
        "d = wl.make_inputs(w, seed=11, device='cuda')\n"
        "out = moe.moe_forward(d['x'], d['logits'], d['w13'], d['w2'], w.k)\n"
        "torch.save(out.cpu(), sys.argv[1])\n")
    outs = []
    for flag in ("1", "0"):
        path = tmp_path / f"out{flag}.pt"
        env = dict(os.environ, MOE_DISABLE_PDL=flag)
        subprocess.run([sys.executable, str(script), str(path)], env=env, check=True, timeout=600)
        outs.append(torch.load(path))
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("T,E,k", [(64, 8, 8), (40, 64, 16), (33, 1024, 16), (16, 1000, 5),
                                   (2, 3, 3)])
def test_fused_path_routing_adversarial(T, E, k):
    """The one-launch path (T <= 64) routes inside its own kernel: all-equal rows,
    signed zeros, -inf and ties at the k-th place give the oracle's ids bit for bit
    and its weights, and the whole output matches the oracle."""
    H, I = 128, 128
    assert moe.moe_forward_fused(T, E, k, H, I)
    w = wl.custom("adv", T, E, k, H, I)
    d = inputs(w, seed=41)
    d["logits"] = adversarial_logits(T, E, seed=T + E).cuda()
    check_full(w, d)


# Shapes for the one-launch FFN + combine (T <= 64): both w2 split choices,
# the multi-launch path's w13 split both on (H >= 512) and off, an odd number
# of 128-row w2 blocks, k = 16 over 1024 experts, one token, the largest routed
# row count (T * k = 1024, full 64-row tiles), and ragged 64-row tiles.
FUSED_SHAPES = [
    ("tiny", None),
    ("decode", None),
    ("skewed_decode", None),
    ("w13_split_only", (8, 16, 2, 1024, 256, 0.0)),
    ("odd_w2_blocks", (8, 32, 4, 384, 256, 0.0)),
    ("many_experts", (40, 1024, 16, 128, 128, 0.0)),
    ("one_token", (1, 4, 2, 256, 128, 0.0)),
    ("full_tiles_k16", (64, 16, 16, 256, 256, 0.0)),   # T*k = 1024, every tile 64 rows
    ("ragged_t33", (33, 64, 4, 512, 384, 0.0)),        # 64-row tiles, ragged; I / 128 = 3
]


def _fused_workload(name, spec):
    if spec is None:
        return wl.WORKLOADS[name]
    T, E, k, H, I, z = spec
    return wl.custom(name, T, E, k, H, I, zipf_s=z)


def test_fused_launch_against_multi_launch_and_oracle(tmp_path):
    """moe_forward's one-launch path (T <= 64) against the multi-launch path
    (MOE_DISABLE_FUSED=1, in a subprocess) and against the oracle.

    Routing outputs are identical.  The one-launch path runs w13 unsplit, so out
    is bit-identical to the multi-launch path wherever that path does too (its
    w13 split needs H >= 512), and otherwise within the parity tolerance."""
    script = tmp_path / "unfused.py"
    script.write_text(
        "import sys, torch\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        f"sys.path.insert(0, {os.path.join(ROOT, 'tests')!r})\n"
        "import mixture_experts_layer_logits_b200 as moe\n"
        "from test_gpu_parity import FUSED_SHAPES, _fused_workload\n"
        "from mixture_experts_layer_logits_b200 import workloads as wl\n"
        "res = {}\n"
        "for name, spec in FUSED_SHAPES:\n"
        "    w = _fused_workload(name, spec)\n"
        "    d = wl.make_inputs(w, seed=13, device='cuda')\n"
        "    assert not moe.moe_forward_fused(w.T, w.E, w.k, w.H, w.I)\n"
        "    res[name] = moe.moe_forward(d['x'], d['logits'], d['w13'], d['w2'], w.k).cpu()\n"
        "torch.save(res, sys.argv[1])\n")
    path = tmp_path / "unfused.pt"
    env = dict(os.environ, MOE_DISABLE_FUSED="1")
    subprocess.run([sys.executable, str(script), str(path)], env=env, check=True, timeout=900)
    ref = torch.load(path)
    for name, spec in FUSED_SHAPES:
        w = _fused_workload(name, spec)
        d = wl.make_inputs(w, seed=13, device="cuda")
        assert moe.moe_forward_fused(w.T, w.E, w.k, w.H, w.I), name
        assert moe.moe_forward_kernel_count(w.T, w.E, w.k, w.H, w.I) == 1, name
        out, ids, wts, off, rows = run_forward(w, d)
        multi = ref[name]
        if w.H < 512:
            assert torch.equal(out.cpu(), multi), name
        else:
            assert_out_close(out, multi.float().numpy().astype(np.float64), what=f"{name} vs multi-launch")
        # the one-launch result against the oracle
        ref_ids, ref_w = oracle.route(host_f32(d["logits"]), w.k)
        assert_routing_equal(ids, wts, ref_ids, ref_w)
        # every token where the oracle is cheap; skewed decode is checked on every
        # token through the same one-launch path by its own test
        small = w.T * w.k * 3 * w.H * w.I <= 4e9
        toks = list(range(w.T)) if small else sorted(set([0, w.T // 2, w.T - 1]))
        w13s, w2s = expert_weights_for(toks, ref_ids, d["w13"], d["w2"])
        want = oracle.forward_tokens(host_bits(d["x"]), host_f32(d["logits"]), w13s, w2s, w.k,
                                     toks, w.I)
        assert_out_close(out[toks], want, what=f"{name} out[{toks}]")
