"""bench.py and __graft_entry__.py read no name they never bind.

Most of bench.py runs only on a GPU, so a name error in one of its measurement
lines would surface only at the end of a GPU run. This check reads the source:
every name a top-level function loads must be bound in that function (its
arguments, assignments, loop and comprehension targets, imports, nested
definitions, exception names), at module level, or among the builtins.
"""
import ast
import builtins
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _module_names(tree):
    names = set(dir(builtins)) | {"__file__", "__name__"}
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            names.add(node.name)
    for node in tree.body:
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names.update((a.asname or a.name).split(".")[0] for a in node.names)
        elif isinstance(node, (ast.Assign, ast.AnnAssign, ast.AugAssign)):
            targets = node.targets if isinstance(node, ast.Assign) else [node.target]
            for t in targets:
                names.update(x.id for x in ast.walk(t) if isinstance(x, ast.Name))
        elif isinstance(node, (ast.If, ast.Try)):
            for sub in ast.walk(node):
                if isinstance(sub, ast.Name) and isinstance(sub.ctx, ast.Store):
                    names.add(sub.id)
                elif isinstance(sub, (ast.Import, ast.ImportFrom)):
                    names.update((a.asname or a.name).split(".")[0] for a in sub.names)
    return names


def _bound_in(fn):
    bound = set()
    for node in ast.walk(fn):
        if isinstance(node, ast.arg):
            bound.add(node.arg)
        elif isinstance(node, ast.Name) and isinstance(node.ctx, (ast.Store, ast.Del)):
            bound.add(node.id)
        elif isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef, ast.ClassDef)):
            bound.add(node.name)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            bound.update((a.asname or a.name).split(".")[0] for a in node.names)
        elif isinstance(node, ast.ExceptHandler) and node.name:
            bound.add(node.name)
        elif isinstance(node, (ast.Global, ast.Nonlocal)):
            bound.update(node.names)
    return bound


def unbound_names(path):
    tree = ast.parse(open(path).read(), path)
    module = _module_names(tree)
    found = []
    for fn in tree.body:
        if not isinstance(fn, (ast.FunctionDef, ast.AsyncFunctionDef)):
            continue
        ok = module | _bound_in(fn)
        for node in ast.walk(fn):
            if isinstance(node, ast.Name) and isinstance(node.ctx, ast.Load) and node.id not in ok:
                found.append(f"{os.path.basename(path)}:{node.lineno} {fn.name}: {node.id}")
    return found


@pytest.mark.parametrize("name", ["bench.py", "__graft_entry__.py"])
def test_no_unbound_names(name):
    assert unbound_names(os.path.join(ROOT, name)) == []


def test_the_check_finds_a_planted_name(tmp_path):
    src = tmp_path / "m.py"
    src.write_text("import os\n\ndef f(a):\n    b = a + 1\n    return roofline[b], os.sep\n")
    assert unbound_names(str(src)) == ["m.py:5 f: roofline"]


def test_clock_sampler_says_why_it_is_silent():
    """Without a GPU (or without NVML and nvidia-smi) the sampler reports the reason
    instead of dropping the clocks key."""
    import bench
    c = bench.ClockSampler(0, period_s=0.01)
    c.start()
    res = c.stop()
    assert isinstance(res, dict)
    assert ("unavailable" in res and res["unavailable"]) or res.get("samples", 0) > 0
