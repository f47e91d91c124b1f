"""Rules the sources keep, checked on the CPU: no cluster-multicast bulk
loads in the CUDA code (every load reads this GPU's own memory through a
plain TMA copy), no path from the package to the oracle (the oracle is test
infrastructure), and every profiling command recorded under profiles/
leaves the GPU clocks alone."""
from __future__ import annotations

import pathlib
import re

ROOT = pathlib.Path(__file__).resolve().parent.parent
PKG = ROOT / "swiglu_backward_int8_b200"


def _cuda_sources():
    return sorted(p for p in (PKG / "csrc").iterdir() if p.suffix in (".cu", ".cuh", ".h"))


def test_cuda_sources_issue_no_multicast_loads():
    assert _cuda_sources()
    for p in _cuda_sources():
        assert ".multicast" not in p.read_text(), p.name   # the PTX qualifier


def test_package_never_reaches_the_oracle():
    files = sorted(PKG.glob("*.py")) + _cuda_sources()
    for p in files:
        text = p.read_text()
        assert not re.search(r"\boracle\b", text), p.name


def _commands(md: str):
    """Shell commands inside the fenced blocks of a markdown file, with
    backslash continuations joined."""
    out = []
    for block in re.findall(r"```[^\n]*\n(.*?)```", md, flags=re.S):
        joined = re.sub(r"\\\n\s*", " ", block)
        out.extend(line.strip() for line in joined.splitlines() if line.strip())
    return out


def test_every_recorded_ncu_run_leaves_the_clocks_alone():
    runs = 0
    for p in sorted((ROOT / "profiles").glob("*.md")):
        for cmd in _commands(p.read_text()):
            for part in re.split(r"&&|;", cmd):
                part = part.strip()
                if not part.startswith("ncu ") or part.startswith("ncu -i "):
                    continue   # reading a report back runs nothing on a GPU
                runs += 1
                assert "--clock-control none" in part, (p.name, part)
    assert runs >= 5
