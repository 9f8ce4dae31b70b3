"""Shared helpers of the parity tests: host copies for the oracle and the layer
output tolerance.

Tolerances (the layer problem statement): integer outputs bit-exact;
topk_weights within 1e-6 absolute; the bf16 layer output within
    max|out - ref| <= 2e-2 * max|ref| + 1e-3   and   sum|out - ref| / sum|ref| <= 5e-3
of the fp64 oracle (the mean relative error read as an L1 ratio, which stays
meaningful where individual reference values are near zero).
"""
import numpy as np
import torch

from mixture_experts_layer_logits_b200 import workloads as wl

WEIGHT_ATOL = 1e-6
OUT_MAX_REL = 2e-2
OUT_MAX_ABS = 1e-3
OUT_MEAN_REL = 5e-3


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().numpy()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return wl.bf16_bits(t)


def out_errors(out: torch.Tensor, ref: np.ndarray):
    got = out.detach().float().cpu().double().numpy()
    err = np.abs(got - ref)
    max_err = float(err.max()) if err.size else 0.0
    max_ref = float(np.abs(ref).max()) if ref.size else 0.0
    denom = float(np.abs(ref).sum())
    mean_rel = float(err.sum() / denom) if denom > 0 else 0.0
    return max_err, max_ref, mean_rel


def assert_out_close(out: torch.Tensor, ref: np.ndarray, what="out"):
    max_err, max_ref, mean_rel = out_errors(out, ref)
    assert max_err <= OUT_MAX_REL * max_ref + OUT_MAX_ABS, (
        f"{what}: max|err| {max_err:.3e} > 2e-2*{max_ref:.3e} + 1e-3")
    assert mean_rel <= OUT_MEAN_REL, f"{what}: mean relative error {mean_rel:.3e} > 5e-3"
    return max_err, mean_rel


def assert_routing_equal(ids, w, ref_ids, ref_w):
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    dw = np.abs(w.cpu().numpy().astype(np.float64) - ref_w.astype(np.float64)).max()
    assert dw <= WEIGHT_ATOL, f"topk_weights differ by {dw:.3e}"


def library_tile_rows(T):
    """Token rows per tile of the grouped GEMMs for T tokens: the smallest power of
    two >= T, between 16 and 256 (each expert's segment is cut into tiles of this
    many rows, the last one ragged)."""
    nt = 16
    while nt < 256 and nt < T:
        nt *= 2
    return nt


def tile_boundary_tokens(expert_offsets, permuted_rows, k, nt):
    """Tokens whose expanded rows are the first or the last row of some nt-row tile
    of some expert's segment: every tile of the grouped GEMMs, its ragged tail
    and every segment boundary then holds at least one checked row."""
    pos = set()
    for e in range(len(expert_offsets) - 1):
        a, b = int(expert_offsets[e]), int(expert_offsets[e + 1])
        for s in range(a, b, nt):
            pos.add(s)
            pos.add(min(s + nt, b) - 1)
    return sorted({int(permuted_rows[p]) // k for p in pos})


def expert_weights_for(tokens, ref_ids, w13, w2):
    """Host copies of only the experts the listed tokens select (per-expert lists)."""
    E = w13.shape[0]
    used = sorted(set(ref_ids[tokens].reshape(-1).tolist()))
    a = [None] * E
    b = [None] * E
    for e in used:
        a[e] = host_bits(w13[e])
        b[e] = host_bits(w2[e])
    return a, b
