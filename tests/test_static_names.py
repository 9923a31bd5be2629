"""Every global name the Python sources read is defined: a module-level binding, an import
or a builtin (a name left over from an edit fails here on the CPU instead of at run time on
a GPU, in a code path the CPU tests cannot execute)."""
import builtins
import os
import symtable

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FILES = sorted(
    [os.path.relpath(os.path.join(d, f), ROOT)
     for sub in ("long_video_diffusion_b200", "oracle", "workloads", "tests")
     for d, _, fs in os.walk(os.path.join(ROOT, sub)) if "__pycache__" not in d
     for f in fs if f.endswith(".py")]
    + ["bench.py", "__graft_entry__.py"])


def _undefined_globals(path):
    src = open(path).read()
    top = symtable.symtable(src, path, "exec")
    defined = {s.get_name() for s in top.get_symbols() if s.is_assigned() or s.is_imported()}
    defined |= set(dir(builtins)) | {"__file__", "__name__", "__doc__", "__spec__"}
    missing = set()

    def walk(t):
        for s in t.get_symbols():
            if t is not top and s.is_referenced() and s.is_global() and s.get_name() not in defined:
                missing.add((t.get_name(), s.get_name()))
        for c in t.get_children():
            walk(c)

    walk(top)
    return missing


@pytest.mark.parametrize("rel", FILES)
def test_no_undefined_global_names(rel):
    assert _undefined_globals(os.path.join(ROOT, rel)) == set()
