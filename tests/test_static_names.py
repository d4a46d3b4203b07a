"""Every name a function of the product's Python files reads resolves: to a
local, an enclosing scope, a module-level name or a builtin. Catches a
renamed argument left behind in a code path the CPU tests cannot run (the
GPU-only wrappers and bench legs) before it costs a GPU run."""

import builtins
import os
import symtable

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = ["rotate_then_quantize_b200/binding.py", "bench.py", "__graft_entry__.py", "kv_synth.py",
         "rotate_then_quantize_b200/build.py"]


def _unresolved(path):
    src = open(os.path.join(ROOT, path)).read()
    top = symtable.symtable(src, path, "exec")
    module_names = {s.get_name() for s in top.get_symbols()
                    if s.is_assigned() or s.is_imported() or s.is_namespace()}
    known = module_names | set(dir(builtins)) | {"__file__", "__name__"}
    bad = []

    def walk(tab, where):
        for child in tab.get_children():
            name = f"{where}.{child.get_name()}"
            for sym in child.get_symbols():
                if sym.is_global() and not sym.is_declared_global() and \
                        sym.get_name() not in known:
                    bad.append((name, sym.get_name()))
            walk(child, name)

    walk(top, path)
    return bad


@pytest.mark.parametrize("path", FILES)
def test_every_free_name_resolves(path):
    assert _unresolved(path) == []
