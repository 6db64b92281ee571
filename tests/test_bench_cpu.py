"""bench.py without a GPU: every function it calls by name is defined, and the
argument parser accepts the driver's command lines."""
import ast
import builtins
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def test_every_called_name_is_defined():
    tree = ast.parse(open(BENCH).read())
    defined = set(dir(builtins))
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)):
            defined.add(node.name)
            if isinstance(node, ast.FunctionDef):      # parameters (callables passed in)
                defined.update(a.arg for a in node.args.args + node.args.kwonlyargs)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            defined.update((a.asname or a.name).split(".")[0] for a in node.names)
        elif isinstance(node, ast.Assign):
            defined.update(t.id for t in node.targets if isinstance(t, ast.Name))
    called = {n.func.id for n in ast.walk(tree) if isinstance(n, ast.Call) and isinstance(n.func, ast.Name)}
    assert called <= defined, sorted(called - defined)


def test_parser_accepts_the_driver_command_lines(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for argv in (["bench.py"], ["bench.py", "--gpus", "8", "--steps", "10", "--warmup", "3"],
                 ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                 ["bench.py", "--no-extra", "--loss", "--no-cpu", "--no-e2e"]):
        monkeypatch.setattr(sys, "argv", argv)
        args = bench.parse()
        assert args.steps >= 1 and args.warmup >= 0
