"""bench.py has code paths that only run on GPUs or under several ranks (the
head-sharded line, the end-to-end pipeline).  This CPU test walks every
function in it and fails on a name that is neither local, a parameter, a
module-level binding nor a builtin, so such a path cannot die on a typo or
a missing import where no CPU test reaches it."""
import ast
import builtins
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _module_names(tree):
    names = set()
    for node in tree.body:
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)):
            names.add(node.name)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            for a in node.names:
                names.add((a.asname or a.name).split(".")[0])
        elif isinstance(node, (ast.Assign, ast.AnnAssign)):
            targets = node.targets if isinstance(node, ast.Assign) else [node.target]
            for t in targets:
                names |= {n.id for n in ast.walk(t) if isinstance(n, ast.Name)}
    return names


def _local_names(fn):
    local = set()
    for n in ast.walk(fn):
        if isinstance(n, (ast.FunctionDef, ast.Lambda)):
            args = n.args
            local |= {a.arg for a in args.args + args.kwonlyargs + args.posonlyargs}
            if args.vararg:
                local.add(args.vararg.arg)
            if args.kwarg:
                local.add(args.kwarg.arg)
            if isinstance(n, ast.FunctionDef):
                local.add(n.name)
        elif isinstance(n, ast.Name) and isinstance(n.ctx, ast.Store):
            local.add(n.id)
        elif isinstance(n, (ast.Import, ast.ImportFrom)):
            local |= {(a.asname or a.name).split(".")[0] for a in n.names}
        elif isinstance(n, ast.ExceptHandler) and n.name:
            local.add(n.name)
    return local


def test_bench_functions_bind_every_name():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    known = _module_names(tree) | set(dir(builtins)) | {"__file__"}
    problems = {}
    # Top-level functions; a nested function's free names are the enclosing function's locals.
    for fn in (n for n in tree.body if isinstance(n, ast.FunctionDef)):
        loads = {n.id for n in ast.walk(fn) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)}
        missing = loads - _local_names(fn) - known
        if missing:
            problems[fn.name] = sorted(missing)
    assert not problems, problems
