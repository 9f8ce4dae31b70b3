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
