"""bench.py's roofline bookkeeping: the committed DRAM traffic stays attached
to the kernel source it was measured on (the key ignores comments and white
space but changes with any code edit), and the algorithmic bytes per launch
add up to the weights a forward streams."""
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
    f = csrc / "attn_split.cu"
    text = f.read_text()
    f.write_text("// a note\n/* a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.source_hash() == h0
    f.write_text(text.replace("kSpKeys = 128", "kSpKeys = 64", 1))
    assert bench.source_hash() != h0


def test_algorithmic_bytes_add_up_to_the_streamed_weights():
    """The per-launch byte counts the roofline uses: the configured figures at
    16 rows, and the weight bytes of one forward's launches (36 layers of the
    four projections plus the LM head) equal the streamed parameter bytes."""
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    import dvlm_gen as gen
    d = gen.QWEN3B
    ab = {k: bench.algorithmic_bytes(k, d, 1344, rows=16) for k in
          ("qkv_gemm", "oproj_gemm", "gateup_gemm", "down_gemm", "lm_head", "attention")}
    assert ab["qkv_gemm"] == 10_633_216 and ab["oproj_gemm"] == 8_585_216
    assert ab["gateup_gemm"] == 90_595_328 and ab["down_gemm"] == 45_572_096
    assert ab["lm_head"] == 622_395_392 and ab["attention"] == 1_523_712
    weights = {k: bench.algorithmic_bytes(k, d, 0, rows=0) for k in ab if k != "attention"}
    assert d.n_layers * sum(v for k, v in weights.items() if k != "lm_head") + weights["lm_head"] == \
        2 * d.streamed_params() == 6_171_394_048
