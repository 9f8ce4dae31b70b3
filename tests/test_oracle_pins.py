"""Pins of the fp64 CPU oracle to facts that do not come from the oracle itself.

* a hand-worked example whose expected values are closed forms (tests/golden);
* routing checked by rank counting (a different algorithm from the oracle's sort);
* invariants of routing and of the permutation;
* special cases that reduce to library routines (torch.softmax for k = E,
  torch.nn.functional.silu + matmul for a one-expert layer);
* a dense loop over all experts masked by the routing weights (no permutation);
* FP8 weights: the E4M3 decoder against the library conversion of all 256 codes,
  bit equality with the bf16 layer on bf16-exact dequantised weights, and a
  dense dequantise-then-multiply loop;
* planted mistakes: a mutated copy of the oracle must fail these pins.
"""
import json
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_logits_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_example.json")


def _f32(v):
    if isinstance(v, str):
        return np.float32(float(v))
    return np.float32(v)


def bf16_bits_from_float(a):
    t = torch.tensor(np.asarray(a, np.float32)).to(torch.bfloat16)
    assert torch.equal(t.float(), torch.tensor(np.asarray(a, np.float32))), "not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def load_hand_example():
    with open(GOLDEN) as f:
        g = json.load(f)
    logits = np.array([[_f32(v) for v in row] for row in g["logits"]], np.float32)
    x = bf16_bits_from_float(g["x"])
    w13 = bf16_bits_from_float(g["w13"])
    w2 = bf16_bits_from_float(g["w2"])
    return g, logits, x, w13, w2


def sigma(z):
    return 1.0 / (1.0 + math.exp(-z))


# ---------------------------------------------------------------- hand example

def test_hand_example_inputs_are_signed_zero_tie():
    g, logits, *_ = load_hand_example()
    assert math.copysign(1.0, logits[2, 0]) == -1.0 and math.copysign(1.0, logits[2, 1]) == 1.0


def test_hand_example_closed_forms_match_stored_numbers():
    g, *_ = load_hand_example()
    e = g["expected"]
    env = dict(exp=math.exp, sigma=sigma)
    for row_f, row_v in zip(e["topk_weights_formula"], e["topk_weights"]):
        for f, v in zip(row_f, row_v):
            assert eval(f, env) == pytest.approx(v, rel=0, abs=1e-15)
    for row_f, row_v in zip(e["out_formula"], e["out"]):
        for f, v in zip(row_f, row_v):
            assert eval(f, env) == pytest.approx(v, rel=0, abs=1e-15)


def test_hand_example_oracle():
    g, logits, x, w13, w2 = load_hand_example()
    e = g["expected"]
    res = oracle.forward(x, logits, w13, w2, g["top_k"])
    np.testing.assert_array_equal(res["topk_ids"], np.array(e["topk_ids"], np.int32))
    np.testing.assert_array_equal(res["expert_offsets"], np.array(e["expert_offsets"], np.int32))
    np.testing.assert_array_equal(res["permuted_rows"], np.array(e["permuted_rows"], np.int32))
    # weights are stored as fp32: compare with the fp32 rounding of the closed forms
    want_w = np.array(e["topk_weights"], np.float64).astype(np.float32)
    np.testing.assert_array_equal(res["topk_weights"], want_w)
    # combine multiplies by the stored fp32 weights, so rebuild the closed forms with them
    s1 = sigma(1.0)
    w = res["topk_weights"].astype(np.float64)
    want_out = np.array([
        [w[0, 0] * 0.0 + w[0, 1] * 0.0, w[0, 0] * 0.0 + w[0, 1] * s1],
        [w[1, 0] * 2 * s1 + w[1, 1] * 0.0, 0.0],
        [w[2, 0] * s1 + w[2, 1] * 4 * s1, -w[2, 0] * s1],
    ])
    np.testing.assert_allclose(res["out"], want_out, rtol=1e-14, atol=1e-15)
    # and, to fp32-weight precision, the pure closed forms
    np.testing.assert_allclose(res["out"], np.array(e["out"]), rtol=1e-7, atol=1e-12)


def test_hand_example_untouched_expert_is_ignored():
    g, logits, x, w13, w2 = load_hand_example()
    base = oracle.forward(x, logits, w13, w2, g["top_k"])["out"]
    w13b = w13.copy()
    w2b = w2.copy()
    w13b[3] = bf16_bits_from_float(np.full((2, 2), 7.0))
    w2b[3] = bf16_bits_from_float(np.full((2, 1), -5.0))
    np.testing.assert_array_equal(oracle.forward(x, logits, w13b, w2b, g["top_k"])["out"], base)


# ---------------------------------------------------------------- routing

def _prefers(la, ea, lb, eb):
    """True if expert ea (logit la) is ranked before expert eb (logit lb)."""
    return la > lb or (la == lb and ea < eb)


def _nasty_logits(rng, T, E):
    vals = np.array([0.0, -0.0, 1.0, -1.0, 0.5, 2.0, -np.inf, 3.25], np.float32)
    a = rng.standard_normal((T, E)).astype(np.float32)
    mask = rng.random((T, E)) < 0.4
    a[mask] = rng.choice(vals, size=mask.sum())
    return a


@pytest.mark.parametrize("T,E,k", [(40, 8, 2), (30, 16, 5), (12, 33, 8), (9, 5, 5), (20, 64, 16)])
def test_route_rank_count_brute_force(T, E, k):
    rng = np.random.default_rng(1000 + E * 17 + k)
    logits = _nasty_logits(rng, T, E)
    logits[0, :] = 0.0                         # an all-equal row
    ids, w = oracle.route(logits, k)
    for t in range(T):
        row = [float(v) for v in logits[t]]
        rank = [sum(_prefers(row[b], b, row[a], a) for b in range(E)) for a in range(E)]
        want = sorted(range(E), key=lambda a: rank[a])[:k]
        assert [int(i) for i in ids[t]] == want
        assert sorted(rank) == list(range(E))      # the key is a strict total order


@pytest.mark.parametrize("T,E,k", [(50, 8, 2), (25, 128, 8), (10, 1024, 8), (7, 3, 1)])
def test_route_invariants(T, E, k):
    rng = np.random.default_rng(7 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32) * 3
    ids, w = oracle.route(logits, k)
    for t in range(T):
        assert len(set(ids[t].tolist())) == k
        assert (ids[t] >= 0).all() and (ids[t] < E).all()
        sel = logits[t, ids[t]]
        assert all(_prefers(float(sel[j]), int(ids[t, j]), float(sel[j + 1]), int(ids[t, j + 1]))
                   for j in range(k - 1))
        assert (w[t] > 0).all()
        assert abs(float(np.sum(w[t].astype(np.float64))) - 1.0) < 4 * k * 6e-8
        # weights are monotone with the logits
        assert all(w[t, j] >= w[t, j + 1] for j in range(k - 1))


def test_route_all_equal_row():
    for E, k in [(8, 2), (128, 8), (1024, 8), (5, 5)]:
        logits = np.full((3, E), 0.25, np.float32)
        ids, w = oracle.route(logits, k)
        np.testing.assert_array_equal(ids, np.tile(np.arange(k, dtype=np.int32), (3, 1)))
        np.testing.assert_array_equal(w, np.full((3, k), np.float32(1.0 / k)))


def test_route_k_equals_E_is_library_softmax():
    rng = np.random.default_rng(3)
    T, E = 16, 12
    logits = (rng.standard_normal((T, E)) * 4).astype(np.float32)
    ids, w = oracle.route(logits, E)
    p = torch.softmax(torch.tensor(logits, dtype=torch.float64), dim=1).numpy()
    for t in range(T):
        np.testing.assert_allclose(w[t].astype(np.float64), p[t, ids[t]], rtol=2e-7, atol=1e-12)
        # descending logit order, stable on equal keys
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
        assert ids[t].tolist() == order


def test_route_softmax_over_selected_equals_renormalised_full_softmax():
    """softmax_sum reading: softmax over all E, keep top-k, divide by their sum."""
    rng = np.random.default_rng(11)
    T, E, k = 32, 64, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = oracle.route(logits, k)
    p = torch.softmax(torch.tensor(logits, dtype=torch.float64), dim=1).numpy()
    for t in range(T):
        sel = p[t, ids[t]]
        np.testing.assert_allclose(w[t].astype(np.float64), sel / sel.sum(), rtol=2e-7)


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (33, 5, 3), (8, 128, 8), (100, 7, 1)])
def test_permute_brute_force_and_invariants(T, E, k):
    rng = np.random.default_rng(T * 31 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    if E > 4:
        logits[:, 2] += 5.0                     # one hot expert
        logits[:, 3] -= 50.0                    # one expert nobody picks
    ids, _ = oracle.route(logits, k)
    off, rows = oracle.permute(ids, E)
    R = T * k
    flat = ids.reshape(-1)
    want = sorted(range(R), key=lambda r: (int(flat[r]), r))
    assert rows.tolist() == want
    assert off[0] == 0 and off[E] == R
    assert all(off[e] <= off[e + 1] for e in range(E))
    assert sorted(rows.tolist()) == list(range(R))
    for e in range(E):
        seg = rows[off[e]:off[e + 1]]
        assert all(flat[r] == e for r in seg)
        assert all(seg[i] < seg[i + 1] for i in range(len(seg) - 1))
        assert off[e + 1] - off[e] == int((flat == e).sum())


# ---------------------------------------------------------------- FFN + combine

def _rand_layer(rng, T, E, k, H, I):
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    w13 = torch.randn(E, 2 * I, H, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    w2 = torch.randn(E, H, I, generator=torch.Generator().manual_seed(int(rng.integers(1 << 30))))
    to_bits = lambda t: t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return logits, to_bits(x), to_bits(w13 / math.sqrt(H)), to_bits(w2 / math.sqrt(I))


def _bits_to_f64(b):
    return torch.tensor(b.view(np.int16)).view(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("T,E,k,H,I", [(5, 6, 3, 8, 4), (9, 4, 4, 16, 8), (12, 10, 2, 32, 24),
                                       (3, 1, 1, 8, 8)])
def test_dense_masked_all_experts_loop(T, E, k, H, I):
    """Every expert on every token, multiplied by its routing weight or 0."""
    rng = np.random.default_rng(T * 100 + E)
    logits, x, w13, w2 = _rand_layer(rng, T, E, k, H, I)
    res = oracle.forward(x, logits, w13, w2, k)
    ids, w = res["topk_ids"], res["topk_weights"]
    X, W13, W2 = _bits_to_f64(x), _bits_to_f64(w13), _bits_to_f64(w2)
    dense = np.zeros((T, H))
    for t in range(T):
        for e in range(E):
            hit = np.nonzero(ids[t] == e)[0]
            m = float(w[t, hit[0]]) if len(hit) else 0.0
            h = W13[e] @ X[t]
            g, u = h[:I], h[I:]
            a = g / (1.0 + np.exp(-g)) * u
            dense[t] += m * (W2[e] @ a)
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-13)


def test_one_expert_layer_is_library_swiglu_mlp():
    """E = 1, k = 1: the layer is the plain SwiGLU MLP w2 . (silu(Wg x) * (Wu x))."""
    rng = np.random.default_rng(5)
    T, H, I = 6, 16, 12
    logits, x, w13, w2 = _rand_layer(rng, T, 1, 1, H, I)
    out = oracle.forward(x, logits, w13, w2, 1)["out"]
    X = torch.tensor(_bits_to_f64(x))
    W13 = torch.tensor(_bits_to_f64(w13))[0]
    W2 = torch.tensor(_bits_to_f64(w2))[0]
    want = torch.nn.functional.silu(X @ W13[:I].T) * (X @ W13[I:].T) @ W2.T
    np.testing.assert_allclose(out, want.numpy(), rtol=1e-12, atol=1e-13)


def test_forward_tokens_matches_forward():
    rng = np.random.default_rng(9)
    T, E, k, H, I = 11, 7, 3, 16, 8
    logits, x, w13, w2 = _rand_layer(rng, T, E, k, H, I)
    full = oracle.forward(x, logits, w13, w2, k)
    toks = [0, 4, 10, 4]
    used = set(full["topk_ids"][toks].reshape(-1).tolist())
    w13s = [w13[e] if e in used else None for e in range(E)]
    w2s = [w2[e] if e in used else None for e in range(E)]
    got = oracle.forward_tokens(x, logits, w13s, w2s, k, toks, I)
    np.testing.assert_array_equal(got, full["out"][toks])
    with pytest.raises(ValueError):
        oracle.forward_tokens(x, logits, [None] * E, [None] * E, k, toks, I)


def _f64_from_f32_bits(bits):
    return np.asarray(bits, np.uint32).view(np.float32).astype(np.float64)


def _bf16_rounding_cases():
    """fp32 bit patterns around bf16 rounding boundaries, plus doubles outside fp32."""
    highs = [0x3F80, 0x3F81, 0x4049, 0x404A, 0x0000, 0x0001, 0x0002, 0x007F, 0x0080, 0x0081,
             0x7F7E, 0x7F7F, 0x1234, 0x5555]
    lows = [0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF]
    bits = [(h << 16) | lo for h in highs for lo in lows]
    bits += [b | 0x80000000 for b in bits]                  # the same, negative
    v = _f64_from_f32_bits(bits).tolist()
    v += [0.0, -0.0, math.inf, -math.inf, 1e300, -1e300, 1e-300, -1e-300,
          1.0 + 2.0 ** -8 + 2.0 ** -30,                     # fp32 rounds it onto a bf16 tie
          float(np.finfo(np.float32).max), 2.0 ** -149, 2.0 ** -133 * 1.5]
    rng = np.random.default_rng(23)
    v += (rng.standard_normal(20000) * np.exp2(rng.integers(-140, 128, 20000))).tolist()
    return np.array(v, np.float64)


def test_round_to_bf16_is_the_library_conversion():
    """The diagnostic rounding equals torch's float64 -> bfloat16 conversion (which
    also goes through fp32 with round-to-nearest-even) bit for bit, on ties with
    even and odd last significand bits, one fp32 ulp either side of a tie,
    subnormals, the overflow boundary, signed zeros, infinities and a random
    spread of magnitudes."""
    v = _bf16_rounding_cases()
    got = oracle.round_to_bf16(v)
    want = torch.tensor(v).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(got.view(np.uint64), want.view(np.uint64))
    # NaNs stay NaN, whatever their payload (an all-ones payload must not carry
    # into the sign bit)
    nans = np.array([0x7FF8000000000000, 0x7FFFFFFFFFFFFFFF, 0xFFFFFFFFFFFFFFFF,
                     0x7FF0000000000001], np.uint64).view(np.float64)
    assert np.isnan(oracle.round_to_bf16(nans)).all()


def test_round_to_bf16_closed_forms():
    """Values fixed by the definition of round-to-nearest-even on an 8-bit significand."""
    ulp1 = 2.0 ** -7                      # bf16 spacing in [1, 2)
    bf16_max = (2.0 - ulp1) * 2.0 ** 127
    cases = [
        (1.0 + ulp1 / 2, 1.0),                        # tie, even neighbour below
        (1.0 + 3 * ulp1 / 2, 1.0 + 2 * ulp1),         # tie, even neighbour above
        (1.0 + ulp1 / 2 + 2.0 ** -20, 1.0 + ulp1),    # just past the tie
        (1.0 + ulp1 / 2 - 2.0 ** -20, 1.0),           # just short of it
        (-(1.0 + 3 * ulp1 / 2), -(1.0 + 2 * ulp1)),
        (bf16_max + 2.0 ** 119, math.inf),            # half an ulp past the largest: tie to inf
        (bf16_max + 2.0 ** 118, bf16_max),
        (2.0 ** -134, 0.0),                           # subnormal tie: 0 (even) and 2^-133 (odd)
        (3 * 2.0 ** -134, 2.0 ** -132),               # tie between 2^-133 (odd) and 2^-132 (even)
        (2.0 ** -135, 0.0),
    ]
    for v, want in cases:
        got = float(oracle.round_to_bf16(np.array([v]))[0])
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), (v, got, want)


def test_round_intermediates_dense_loop():
    """round_intermediates = True against a dense all-experts loop that rounds act
    and y to bf16 with the library conversion (no permutation, no gather)."""
    rng = np.random.default_rng(29)
    T, E, k, H, I = 7, 5, 2, 16, 8
    logits, x, w13, w2 = _rand_layer(rng, T, E, k, H, I)
    res = oracle.forward(x, logits, w13, w2, k, round_intermediates=True)
    ids, w = res["topk_ids"], res["topk_weights"]
    X, W13, W2 = _bits_to_f64(x), _bits_to_f64(w13), _bits_to_f64(w2)
    bf = lambda a: torch.tensor(a).to(torch.bfloat16).double().numpy()
    dense = np.zeros((T, H))
    for t in range(T):
        for e in range(E):
            hit = np.nonzero(ids[t] == e)[0]
            m = float(w[t, hit[0]]) if len(hit) else 0.0
            h = W13[e] @ X[t]
            g, u = h[:I], h[I:]
            dense[t] += m * bf(W2[e] @ bf(g / (1.0 + np.exp(-g)) * u))
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-13)
    exact = oracle.forward(x, logits, w13, w2, k)["out"]
    assert not np.array_equal(res["out"], exact)


def test_round_intermediates_stays_within_bf16_error():
    rng = np.random.default_rng(21)
    T, E, k, H, I = 8, 4, 2, 64, 32
    logits, x, w13, w2 = _rand_layer(rng, T, E, k, H, I)
    exact = oracle.forward(x, logits, w13, w2, k)["out"]
    rounded = oracle.forward(x, logits, w13, w2, k, round_intermediates=True)["out"]
    assert np.abs(rounded - exact).max() <= 2e-2 * np.abs(exact).max()
    assert not np.array_equal(rounded, exact)


def test_oracle_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 3), np.float32), 4)            # k > E
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 5]], np.int32), 4)          # expert id out of range


def test_workload_inputs_deterministic_and_shaped():
    w = wl.WORKLOADS["tiny"]
    a = wl.make_inputs(w, seed=0)
    b = wl.make_inputs(w, seed=0)
    for key in a:
        assert torch.equal(a[key], b[key])
    assert a["logits"].shape == (16, 8) and a["logits"].dtype == torch.float32
    assert a["x"].shape == (16, 256) and a["x"].dtype == torch.bfloat16
    assert a["w13"].shape == (8, 1024, 256) and a["w2"].shape == (8, 256, 512)
    std13 = a["w13"].float().std().item()
    assert abs(std13 - 1 / 16) < 0.01 * 1 / 16 * 10
    rs = wl.custom("rs", 512, 64, 8, dup_frac=0.05)
    lg = wl.make_logits(rs)
    dups = sum(len(r) - len(np.unique(r)) for r in lg.numpy())
    assert dups > 0.5 * 0.05 * 512 * 64
    z = wl.zipf_bias(256, 1.2)
    assert z[0] > z[1] > z[255]
    assert abs(float(torch.exp(z.double() / 2).sum()) - 1.0) < 1e-6


# ---------------------------------------------------------------- FP8 (E4M3) weights

def _rand_w8_layer(rng, T, E, k, H, I, pow2_scales):
    """Random E4M3 codes (no NaN codes) and positive per-row scales."""
    logits, x, _, _ = _rand_layer(rng, T, E, k, H, I)

    def codes(shape):
        q = rng.integers(0, 256, shape, dtype=np.uint8)
        q[(q & 0x7F) == 0x7F] = 0x7E  # NaN codes -> 448 of the same sign
        return q

    def scales(shape):
        if pow2_scales:
            return (2.0 ** rng.integers(-9, -3, shape)).astype(np.float32)
        return rng.uniform(1e-3, 1e-2, shape).astype(np.float32)

    return (logits, x, codes((E, 2 * I, H)), scales((E, 2 * I)), codes((E, H, I)),
            scales((E, H)))


def _e4m3_library(q):
    return torch.from_numpy(np.ascontiguousarray(q)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decoder_is_the_library_conversion():
    """Every one of the 256 codes decodes to PyTorch's float8_e4m3fn value."""
    q = np.arange(256, dtype=np.uint8)
    got, want = oracle.e4m3_to_float64(q), _e4m3_library(q)
    nan = np.isnan(want)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.isnan(got[nan]).all()
    np.testing.assert_array_equal(got[~nan], want[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x80] == 0.0


@pytest.mark.parametrize("T,E,k,H,I", [(5, 6, 3, 8, 4), (9, 4, 4, 16, 8), (3, 1, 1, 8, 8)])
def test_w8_layer_equals_bf16_layer_on_bf16_exact_weights(T, E, k, H, I):
    """With power-of-two scales every dequantised weight is a bf16 value, and the
    FP8 layer must equal the bf16 layer on those weights bit for bit."""
    rng = np.random.default_rng(T * 7 + E)
    logits, x, q13, s13, q2, s2 = _rand_w8_layer(rng, T, E, k, H, I, pow2_scales=True)
    w13 = _e4m3_library(q13) * s13[..., None]
    w2 = _e4m3_library(q2) * s2[..., None]
    to_bits = lambda a: torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    b13, b2 = to_bits(w13), to_bits(w2)
    np.testing.assert_array_equal(_bits_to_f64(b13), w13)  # the premise: exact in bf16
    ref = oracle.forward(x, logits, b13, b2, k)
    got = oracle.forward_w8(x, logits, q13, s13, q2, s2, k)
    for key in ("topk_ids", "topk_weights", "expert_offsets", "permuted_rows", "out"):
        np.testing.assert_array_equal(got[key], ref[key])


@pytest.mark.parametrize("T,E,k,H,I", [(5, 6, 3, 8, 4), (12, 10, 2, 32, 24)])
def test_w8_dense_dequantised_loop(T, E, k, H, I):
    """Arbitrary scales: every expert on every token with weights dequantised by
    the library (code value * row scale), masked by the routing weights."""
    rng = np.random.default_rng(T * 13 + E)
    logits, x, q13, s13, q2, s2 = _rand_w8_layer(rng, T, E, k, H, I, pow2_scales=False)
    res = oracle.forward_w8(x, logits, q13, s13, q2, s2, k)
    ids, w = res["topk_ids"], res["topk_weights"]
    X = _bits_to_f64(x)
    W13 = _e4m3_library(q13) * s13.astype(np.float64)[..., None]
    W2 = _e4m3_library(q2) * s2.astype(np.float64)[..., None]
    dense = np.zeros((T, H))
    for t in range(T):
        for e in range(E):
            hit = np.nonzero(ids[t] == e)[0]
            m = float(w[t, hit[0]]) if len(hit) else 0.0
            h = W13[e] @ X[t]
            g, u = h[:I], h[I:]
            dense[t] += m * (W2[e] @ (g / (1.0 + np.exp(-g)) * u))
    np.testing.assert_allclose(res["out"], dense, rtol=1e-12, atol=1e-13)


def test_w8_forward_tokens_matches_forward_w8():
    rng = np.random.default_rng(17)
    T, E, k, H, I = 11, 7, 3, 16, 8
    logits, x, q13, s13, q2, s2 = _rand_w8_layer(rng, T, E, k, H, I, pow2_scales=False)
    full = oracle.forward_w8(x, logits, q13, s13, q2, s2, k)["out"]
    toks = [0, 4, 10]
    experts = [(q13[e], s13[e], q2[e], s2[e]) for e in range(E)]
    sel = oracle.forward_tokens_w8(x, logits, experts, k, toks, I)
    np.testing.assert_array_equal(sel, full[toks])


def test_workload_w8_quantisation_reconstructs_weights():
    w = wl.custom("q", 4, 3, 2, 256, 128)
    q13, s13, q2, s2 = wl.make_weights_w8(w)
    w13, w2 = wl.make_weights(w)
    for q, sc, ref in ((q13, s13, w13), (q2, s2, w2)):
        deq = _e4m3_library(q.numpy()) * sc.double().numpy()[..., None]
        r = ref.double().numpy()
        # E4M3 keeps 3 mantissa bits: round-to-nearest error <= 2^-4 relative, and
        # every row's largest magnitude maps to 448 exactly
        np.testing.assert_array_less(np.abs(deq - r), 2.0 ** -4 * np.abs(r) + 2.0 ** -9 * sc.double().numpy()[..., None] + 1e-12)
        np.testing.assert_allclose(np.abs(deq).max(axis=-1), np.abs(r).max(axis=-1), rtol=1e-6)


# ---------------------------------------------------------------- planted mistakes

MUTATIONS = [
    ("swap gate and up",
     "const double silu = gate / (1.0 + exp(-gate));\n        act[c] = silu * up;",
     "const double silu = up / (1.0 + exp(-up));\n        act[c] = silu * gate;"),
    ("tie goes to the higher index",
     "return (a->expert < b->expert) ? -1 : (a->expert > b->expert) ? 1 : 0;",
     "return (a->expert > b->expert) ? -1 : (a->expert < b->expert) ? 1 : 0;"),
    ("token map r % T instead of r / k",
     "const long t = r / k;                  /* expanded id -> token */",
     "const long t = r % T;"),
    ("softmax over the top-1 only",
     "for (int j = 0; j < k; ++j) denom += exp(scratch[j].logit - lmax);",
     "for (int j = 0; j < 1; ++j) denom += exp(scratch[j].logit - lmax);"),
    ("unstable scatter (descending r)",
     "for (long r = 0; r < R; ++r) permuted_rows[cursor[topk_ids[r]]++] = (int32_t)r;",
     "for (long r = R - 1; r >= 0; --r) permuted_rows[cursor[topk_ids[r]]++] = (int32_t)r;"),
    ("combine drops the last choice",
     "for (int j = 0; j < k; ++j)\n                acc += (double)topk_weights",
     "for (int j = 0; j + 1 < k; ++j)\n                acc += (double)topk_weights"),
    ("E4M3 exponent bias 8",
     "ldexp(1.0 + m / 8.0, e - 7)",
     "ldexp(1.0 + m / 8.0, e - 8)"),
    ("FP8 gate and up scales swapped",
     "const double sg = s13_e[c], su = s13_e[I + c];",
     "const double sg = s13_e[I + c], su = s13_e[c];"),
    ("bf16 rounding truncates",
     "u += 0x7fffu + lsb;",
     "(void)lsb;"),
    ("bf16 rounding ties away from zero",
     "u += 0x7fffu + lsb;",
     "u += 0x8000u; (void)lsb;"),
    ("bf16 rounding drops the finite test (NaN/inf carry)",
     "if ((u & 0x7f800000u) != 0x7f800000u) {          /* finite */",
     "if (1) {"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(name, old, new, monkeypatch, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")).read()
    assert old in src, f"mutation anchor for '{name}' not found"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", str(so),
                    str(mut), "-lm"], check=True)
    import ctypes

    saved = oracle._lib
    try:
        oracle._lib = None
        monkeypatch.setattr(oracle, "_LIB_PATH", str(so))
        caught = False
        for check in (test_hand_example_oracle,
                      lambda: test_route_rank_count_brute_force(40, 8, 2),
                      lambda: test_permute_brute_force_and_invariants(33, 5, 3),
                      lambda: test_dense_masked_all_experts_loop(5, 6, 3, 8, 4),
                      test_e4m3_decoder_is_the_library_conversion,
                      lambda: test_w8_dense_dequantised_loop(5, 6, 3, 8, 4),
                      test_round_to_bf16_is_the_library_conversion,
                      test_round_to_bf16_closed_forms,
                      test_round_intermediates_dense_loop):
            try:
                check()
            except AssertionError:
                caught = True
        assert caught, f"planted mistake '{name}' passed every pin"
    finally:
        oracle._lib = saved
