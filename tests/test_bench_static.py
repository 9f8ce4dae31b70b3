"""bench.py's GPU-only code paths cannot run here, so check statically that every
function in it refers only to names that exist (its own locals, enclosing
scopes, module-level definitions and imports, or builtins)."""
import builtins
import os
import symtable

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _undefined_globals(path):
    src = open(path).read()
    top = symtable.symtable(src, os.path.basename(path), "exec")
    defined = {s.get_name() for s in top.get_symbols() if s.is_assigned() or s.is_imported()}
    defined |= set(dir(builtins))
    bad = []

    def walk(table):
        for child in table.get_children():
            for sym in child.get_symbols():
                if sym.is_referenced() and sym.is_global() and sym.get_name() not in defined:
                    bad.append(f"{child.get_name()}: {sym.get_name()}")
            walk(child)

    walk(top)
    return bad


def test_bench_refers_only_to_defined_names():
    assert _undefined_globals(os.path.join(ROOT, "bench.py")) == []


def test_graft_entry_refers_only_to_defined_names():
    assert _undefined_globals(os.path.join(ROOT, "__graft_entry__.py")) == []


def test_stage_work_counts_e4m3_weights_at_one_byte_plus_row_scales():
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_logits_b200 import workloads as wl

    w = wl.WORKLOADS["decode"]
    n = 54
    bf = bench.stage_work(w, n)
    f8 = bench.stage_work(w, n, "e4m3")
    T, k, H, I = w.T, w.k, w.H, w.I
    # x, routing weights and rows, out; the routing's logits and outputs
    rest = T * H * 2 + T * k * 8 + T * H * 2 + T * w.E * 4 + T * k * 12 + (w.E + 1) * 4
    assert bf["fused_ffn"]["bytes"] == n * 3 * I * H * 2 + rest
    assert f8["fused_ffn"]["bytes"] == n * (3 * I * H + (2 * I + H) * 4) + rest
    assert f8["fused_ffn"]["flops"] == bf["fused_ffn"]["flops"]  # same bf16 products
    assert f8["route_permute"] == bf["route_permute"] and f8["combine"] == bf["combine"]


def test_traffic_table_keys_name_real_workloads_and_stages():
    """Every measured DRAM-bytes entry is keyed by a workload the bench knows (with
    "+e4m3" for E4M3 weights) and a stage its roofline can pick, and the
    dominant kernel of every suite record but the tiny layer has one."""
    import sys

    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_logits_b200 import workloads as wl

    stages = set(bench.stage_work(wl.WORKLOADS["decode"], 1)) | {"route"}
    for (tag, stage), traffic in bench.NCU_TRAFFIC.items():
        name, _, fmt = tag.partition("+")
        assert name in wl.WORKLOADS and fmt in ("", "e4m3"), tag
        assert stage in stages, stage
        assert isinstance(traffic, int) and traffic > 0
    for name, fmt in [("prefill", "bf16")] + bench.SUITE:
        if name == "tiny":
            continue
        stage = {"prefill": "w13", "routing_stress": "route"}.get(name, "fused_ffn")
        tag = name + ("+e4m3" if fmt == "e4m3" else "")
        assert (tag, stage) in bench.NCU_TRAFFIC, (tag, stage)
