"""Static checks of bench.py that need no GPU: every attribute a step class reads through `self`
is assigned (or defined) in that class, so a workload cannot fail on a missing attribute only
once it runs on a GPU."""
import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_step_classes_define_every_attribute_they_read():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    problems = []
    for cls in [n for n in tree.body if isinstance(n, ast.ClassDef)]:
        defined = set()
        for node in cls.body:
            if isinstance(node, (ast.FunctionDef, ast.AsyncFunctionDef)):
                defined.add(node.name)
            elif isinstance(node, ast.Assign):
                defined.update(t.id for t in node.targets if isinstance(t, ast.Name))
            elif isinstance(node, ast.AnnAssign) and isinstance(node.target, ast.Name):
                defined.add(node.target.id)
        reads = []
        for node in ast.walk(cls):
            if isinstance(node, ast.Attribute) and isinstance(node.value, ast.Name) and node.value.id == "self":
                if isinstance(node.ctx, ast.Store):
                    defined.add(node.attr)
                else:
                    reads.append((node.attr, node.lineno))
            elif isinstance(node, (ast.Assign, ast.AugAssign)):
                targets = node.targets if isinstance(node, ast.Assign) else [node.target]
                for t in targets:
                    for el in (t.elts if isinstance(t, ast.Tuple) else [t]):
                        if isinstance(el, ast.Attribute) and isinstance(el.value, ast.Name) and el.value.id == "self":
                            defined.add(el.attr)
        problems += [(cls.name, a, ln) for a, ln in reads if a not in defined]
    assert not problems, problems
