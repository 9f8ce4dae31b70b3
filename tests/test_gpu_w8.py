"""FP8 (E4M3) expert weights: moe_forward_w8 on the GPU against the oracle's
forward_w8 / forward_tokens_w8 (weight = e4m3(code) * per-row scale, fp64).

Routing outputs are bit-exact as everywhere; the layer output is held to the
same tolerance as the bf16 path, against the oracle's exact dequantised
weights (the codes and scales themselves are the inputs, so quantisation error
is not part of the comparison).
"""
import numpy as np
import pytest
import torch

import oracle
import mixture_experts_layer_logits_b200 as moe
from mixture_experts_layer_logits_b200 import workloads as wl

from parity import assert_out_close, assert_routing_equal, host_bits, host_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    moe.load_library()


def w8_inputs(w, seed=0):
    d = wl.make_inputs(w, seed=seed, device="cuda", weights=False)
    d["q13"], d["s13"], d["q2"], d["s2"] = wl.make_weights_w8(w, seed=seed, device="cuda")
    return d


def run_w8(w, d, events=None):
    T, E, k = w.T, w.E, w.k
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wts = torch.empty(T, k, dtype=torch.float32, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    rows = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = moe.workspace(T, E, k, w.H, w.I)
    out = moe.moe_forward_w8(d["x"], d["logits"], d["q13"], d["s13"], d["q2"], d["s2"], k, ws=ws,
                             topk_ids=ids, topk_weights=wts, expert_offsets=off,
                             permuted_rows=rows, events=events)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == moe.MOE_OK
    return out, ids, wts, off, rows


def host_u8(t):
    return t.detach().to("cpu").contiguous().numpy()


SHAPES = [
    # name, T, E, k, H, I, zipf  (all within the one-launch FFN's range)
    ("tiny", None),
    ("decode", None),
    ("one_token", (1, 4, 2, 256, 128, 0.0)),
    ("odd_w2_blocks", (8, 32, 4, 384, 256, 0.0)),      # H / 128 odd: a half w2 block pair
    ("w13_long_k", (8, 16, 2, 1024, 256, 0.0)),
    ("full_tiles_k16", (64, 16, 16, 256, 256, 0.0)),   # every tile 64 rows
    ("ragged_t33", (33, 64, 4, 512, 384, 0.0)),        # ragged 64-row tiles, I / 128 = 3
    ("nt32", (17, 16, 4, 256, 256, 0.0)),
    ("hot_expert", (48, 64, 4, 512, 256, 2.5)),        # most experts empty
    ("many_experts", (40, 1024, 16, 128, 128, 0.0)),
]


def _workload(name, spec):
    if spec is None:
        return wl.WORKLOADS[name]
    T, E, k, H, I, z = spec
    return wl.custom(name, T, E, k, H, I, zipf_s=z)


@pytest.mark.parametrize("name,spec", SHAPES, ids=[s[0] for s in SHAPES])
def test_forward_w8_matches_oracle(name, spec):
    w = _workload(name, spec)
    assert moe.moe_forward_w8_supported(w.T, w.E, w.k, w.H, w.I)
    d = w8_inputs(w, seed=3)
    out, ids, wts, off, rows = run_w8(w, d)
    ref = oracle.forward_w8(host_bits(d["x"]), host_f32(d["logits"]), host_u8(d["q13"]),
                            host_f32(d["s13"]), host_u8(d["q2"]), host_f32(d["s2"]), w.k)
    assert_routing_equal(ids, wts, ref["topk_ids"], ref["topk_weights"])
    np.testing.assert_array_equal(off.cpu().numpy(), ref["expert_offsets"])
    np.testing.assert_array_equal(rows.cpu().numpy(), ref["permuted_rows"])
    assert_out_close(out, ref["out"], what=f"{name} out")


def test_forward_w8_skewed_decode_all_tokens():
    """The full skewed-decode shape (T=64, E=256, k=8, H=7168, I=2048) on every
    token: the oracle gets only the experts the tokens select."""
    w = wl.WORKLOADS["skewed_decode"]
    d = w8_inputs(w, seed=0)
    out, ids, wts, off, rows = run_w8(w, d)
    ref_ids, ref_w = oracle.route(host_f32(d["logits"]), w.k)
    assert_routing_equal(ids, wts, ref_ids, ref_w)
    ref_off, ref_rows = oracle.permute(ref_ids, w.E)
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(rows.cpu().numpy(), ref_rows)
    toks = list(range(w.T))
    experts = [None] * w.E
    for e in sorted(set(ref_ids.reshape(-1).tolist())):
        experts[e] = (host_u8(d["q13"][e]), host_f32(d["s13"][e]), host_u8(d["q2"][e]),
                      host_f32(d["s2"][e]))
    want = oracle.forward_tokens_w8(host_bits(d["x"]), host_f32(d["logits"]), experts, w.k, toks,
                                    w.I)
    assert_out_close(out, want, what="out (all 64 tokens)")
    del d
    torch.cuda.empty_cache()


def test_forward_w8_is_deterministic_and_timed_variant_identical():
    w = wl.WORKLOADS["decode"]
    d = w8_inputs(w, seed=5)
    a = run_w8(w, d)[0].clone()
    b = run_w8(w, d)[0].clone()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for e in ev:  # torch creates the CUDA event on its first record
        e.record()
    c = run_w8(w, d, events=ev)[0]
    assert torch.equal(a, b) and torch.equal(a, c)
    assert ev[0].elapsed_time(ev[4]) > 0


def test_forward_w8_scales_enter_per_row():
    """The scales are read per expert and weight row: doubling expert 0's w2 row
    scales (every token routes to both experts, k = E = 2) changes the output and
    still matches the oracle given the same scales."""
    w = wl.custom("two_experts", 16, 2, 2, 256, 128)
    d = w8_inputs(w, seed=9)
    base = run_w8(w, d)[0].double()
    d2 = dict(d)
    d2["s2"] = d["s2"].clone()
    d2["s2"][0] *= 2
    twice = run_w8(w, d2)[0].double()
    ref = oracle.forward_w8(host_bits(d["x"]), host_f32(d["logits"]), host_u8(d["q13"]),
                            host_f32(d["s13"]), host_u8(d["q2"]), host_f32(d2["s2"]), w.k)
    assert_out_close(twice.to(torch.bfloat16), ref["out"], what="w2 scale of expert 0 doubled")
    assert not torch.equal(base, twice)


def test_forward_w8_rejects_bf16_weights_and_wrong_scales():
    w = wl.WORKLOADS["tiny"]
    d = w8_inputs(w)
    with pytest.raises(ValueError):
        moe.moe_forward_w8(d["x"], d["logits"], d["q13"].view(torch.int8), d["s13"], d["q2"],
                           d["s2"], w.k)
    with pytest.raises(ValueError):
        moe.moe_forward_w8(d["x"], d["logits"], d["q13"], d["s13"][:, :-1], d["q2"], d["s2"],
                           w.k)


def test_forward_w8_rows_of_different_magnitudes():
    """Token rows scaled by powers of two from 2^-40 to 2^40, one row all zero and
    one holding a few large entries among tiny ones: each token's output is
    checked against the oracle on its own scale (the layer is linear in each
    x row up to SwiGLU, so a wrong per-row operand scale shows in that row)."""
    w = wl.custom("row_scales", 16, 16, 4, 512, 256)
    d = w8_inputs(w, seed=11)
    x = d["x"].float()
    exps = [-40, -30, -24, -12, -6, -1, 0, 1, 3, 7, 12, 20, 30, 40, 0, 0]
    for t, e in enumerate(exps):
        x[t] *= 2.0 ** e
    x[14] = 0.0
    x[15] *= 2.0 ** -30
    x[15, ::97] = 3.0  # a handful of entries 2^30 above the rest
    d["x"] = x.to(torch.bfloat16)
    out, ids, wts, off, rows = run_w8(w, d)
    ref = oracle.forward_w8(host_bits(d["x"]), host_f32(d["logits"]), host_u8(d["q13"]),
                            host_f32(d["s13"]), host_u8(d["q2"]), host_f32(d["s2"]), w.k)
    assert_routing_equal(ids, wts, ref["topk_ids"], ref["topk_weights"])
    got = out.float().cpu().double().numpy()
    assert np.all(got[14] == 0.0)
    for t in range(w.T):
        if t == 14:
            continue
        r = ref["out"][t]
        scale = np.abs(r).max()
        assert scale > 0 and np.isfinite(scale), t
        err = np.abs(got[t] - r).max()
        assert err <= 2e-2 * scale, f"token {t}: max|err| {err:.3e} vs max|ref| {scale:.3e}"
        assert np.abs(got[t] - r).sum() <= 5e-3 * np.abs(r).sum(), f"token {t}: mean error"
