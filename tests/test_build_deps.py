"""The library is rebuilt when any file it is compiled from changes: every
local #include reached from the sources is among the rebuild dependencies
(CPU only)."""
import os
import re

from mqa_attention_attn_b200 import build


def _local_includes(path, seen):
    for name in re.findall(r'#include\s+"([^"]+)"', open(path).read()):
        dep = os.path.normpath(os.path.join(os.path.dirname(path), name))
        if dep not in seen:
            seen.add(dep)
            _local_includes(dep, seen)
    return seen


def test_every_included_file_is_a_rebuild_dependency():
    deps = set(os.path.normpath(d) for d in build._deps())
    deps.add(os.path.normpath(os.path.join(build.ROOT, "include", "attn.h")))
    reached = set()
    for src in build.SOURCES:
        path = os.path.normpath(os.path.join(build.CSRC, src))
        reached.add(path)
        _local_includes(path, reached)
    assert reached, "no sources"
    missing = sorted(reached - deps)
    assert not missing, f"not checked for staleness: {missing}"
    assert any(p.endswith("rope.cuh") for p in reached)
