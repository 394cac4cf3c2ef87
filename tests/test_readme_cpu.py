"""The README's usage example stays in step with the binding: it parses, and
every binding call in it binds to the function's signature."""
from __future__ import annotations

import ast
import inspect
import os

from weight_only_quantized_bcq_b200 import lutgemm

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _example() -> str:
    text = open(os.path.join(ROOT, "README.md"), encoding="utf-8").read()
    block = text[text.index("## Use (Python binding)"):text.index("Every call is asynchronous")]
    return "\n".join(line[4:] for line in block.splitlines() if line.startswith("    "))


def test_readme_example_calls_match_the_binding():
    tree = ast.parse(_example())
    calls = [n for n in ast.walk(tree) if isinstance(n, ast.Call) and isinstance(n.func, ast.Attribute)
             and isinstance(n.func.value, ast.Name) and n.func.value.id == "lutgemm"]
    assert {c.func.attr for c in calls} >= {"fit_bcq", "pack_bcq", "pack_scales", "new_workspace", "run"}
    for c in calls:
        sig = inspect.signature(getattr(lutgemm, c.func.attr))
        sig.bind(*[None] * len(c.args), **{k.arg: None for k in c.keywords})
