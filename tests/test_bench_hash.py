"""bench.py ties the ncu counters in profiles/ to a hash of the kernels' code
with comments removed: editing a comment keeps the hash (the counters still
describe the kernel), editing code changes it (the counters are dropped)."""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _hash_of(tmp_path, monkeypatch, text: str) -> str:
    import bench
    csrc = tmp_path / "weight_only_quantized_bcq_b200" / "csrc"
    csrc.mkdir(parents=True, exist_ok=True)
    (csrc / "k.cu").write_text(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench._code_hash(("k.cu",))


def test_code_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    base = "// header\n__global__ void k(int* p) {\n  p[0] = 1;  /* one */\n}\n"
    h0 = _hash_of(tmp_path, monkeypatch, base)
    assert _hash_of(tmp_path, monkeypatch, base.replace("// header", "// another header\n// more")) == h0
    assert _hash_of(tmp_path, monkeypatch, base.replace("/* one */", "/* the value one,\n  on two lines */")) == h0
    assert _hash_of(tmp_path, monkeypatch, base.replace("p[0] = 1;", "p[0] = 2;")) != h0
    assert _hash_of(tmp_path, monkeypatch, base.replace("int* p", "int* q").replace("p[0]", "q[0]")) != h0
