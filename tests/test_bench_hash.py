"""bench.py attaches the committed DRAM traffic to the kernel source it was
measured on: the key ignores comments and white space but changes with any
code edit."""
import importlib
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture()
def bench_copy(tmp_path, monkeypatch):
    dst = tmp_path / "block_diffusion_vlm_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "block_diffusion_vlm_b200", "csrc"), dst)
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return bench, dst


def test_traffic_key_covers_only_the_kernels_sources(bench_copy):
    bench, csrc = bench_copy
    h0 = bench.source_hash(bench.TRAFFIC_SOURCES["lm_head"])
    f = csrc / "spec.cu"
    f.write_text(f.read_text() + "\nstatic int unrelated_edit;\n")
    assert bench.source_hash(bench.TRAFFIC_SOURCES["lm_head"]) == h0
    f = csrc / "lmhead.cu"
    f.write_text(f.read_text() + "\nstatic int related_edit;\n")
    assert bench.source_hash(bench.TRAFFIC_SOURCES["lm_head"]) != h0


def test_source_hash_ignores_comments_but_not_code(bench_copy):
    bench, csrc = bench_copy
    h0 = bench.source_hash()
    f = csrc / "attn.cu"
    text = f.read_text()
    f.write_text("// a note\n/* a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.source_hash() == h0
    f.write_text(text.replace("kChunk = 64", "kChunk = 32", 1))
    assert bench.source_hash() != h0
