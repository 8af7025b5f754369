"""The seeded input generator serves both the oracle and the CUDA path; these
checks hold it to the stated input recipe: reproducible per tensor name,
independent across names, exact bf16 storage values, the configured shapes
and distributions, and speculative-accept inputs whose agreeing prefix is
known by construction."""
import numpy as np
import pytest
import torch

import dvlm_gen as gen


def test_streams_are_reproducible_and_independent():
    a = gen.normal(3, "layer0.wq", (64, 32))
    assert np.array_equal(a, gen.normal(3, "layer0.wq", (64, 32)))
    assert not np.array_equal(a, gen.normal(3, "layer0.wk", (64, 32)))
    assert not np.array_equal(a, gen.normal(4, "layer0.wq", (64, 32)))
    # regenerating one tensor alone gives the same values as in any other order
    gen.normal(3, "embed", (10, 10))
    assert np.array_equal(a, gen.normal(3, "layer0.wq", (64, 32)))
    b = gen.normal(3, "layer0.wk", (64, 32))
    assert abs(float(np.corrcoef(a.ravel(), b.ravel())[0, 1])) < 0.05


def test_bf16_storage_values_are_exact():
    t, vals = gen.normal_bf16(1, "x", (257, 33), 0.02)
    assert t.dtype == torch.bfloat16 and vals.dtype == np.float32
    assert np.array_equal(vals, t.float().numpy())
    raw = gen.normal(1, "x", (257, 33), 0.02)
    # round to nearest even from fp32: within half a bf16 ulp of the draw
    ulp = 2.0 ** (np.floor(np.log2(np.abs(raw.astype(np.float64)))) - 7)
    assert np.all(np.abs(vals.astype(np.float64) - raw) <= ulp / 2)


def test_distributions_and_scales():
    d = gen.QWEN3B
    _, w = gen.layer_weight(d, 4, 0, "wq")
    assert w.shape == (d.n_q_heads * d.head_dim, d.hidden)
    assert abs(float(w.std()) - 0.02) < 0.001 and abs(float(w.mean())) < 0.001
    _, lm = gen.lmhead_case(2, 16, H=256, V=4096, second_set=False)[1]
    assert abs(float(lm.std()) - 0.02 * 25) < 0.01
    shapes = {n: gen.layer_weight(gen.TINY, 0, 0, n)[1].shape for n in gen.layer_weight_names()}
    assert shapes == {"wq": (32, 32), "wk": (16, 32), "wv": (16, 32), "wo": (32, 32), "wg": (64, 32),
                      "wu": (64, 32), "wd": (32, 64)}
    assert gen.TINY.n_params() == sum(int(np.prod(s)) for s in shapes.values()) + 2 * 256 * 32
    # a forward streams every decoder matrix and the LM head (6.171 GB in bf16), not the embedding table
    assert gen.QWEN3B.streamed_params() == 3_085_697_024
    assert gen.QWEN3B.n_params() == 3_085_697_024 + 151936 * 2048


def test_decode_context_recipe():
    d = gen.QWEN3B
    vis_t, vis, ids = gen.decode_context(d, 4, 1280, 64)
    assert vis.shape == (1280, 2048) and vis_t.dtype == torch.bfloat16
    assert abs(float(vis.std()) - 1.0) < 0.01
    assert ids.shape == (64,) and ids.dtype == np.int32
    assert ids.min() >= 0 and ids.max() < d.vocab - 1          # [MASK] = V-1 is never a context id
    _, _, ids2 = gen.decode_context(gen.TINY, 0, 32, 16, 16)
    assert len(ids2) == 32 and ids2.max() < gen.TINY.mask_id


@pytest.mark.parametrize("b", [1, 8])
def test_spec_case_plants_the_agreeing_prefix(b):
    B, V = 16, 4096
    t, vals, top, draft, k = gen.spec_case(5, b, B, V)
    assert vals.shape == (b, B, V) and t.dtype == torch.bfloat16
    assert np.array_equal(vals.argmax(axis=-1), top)          # the planted id is every row's top-1
    for i in range(b):
        assert 0 <= k[i] <= B
        assert np.array_equal(draft[i, :k[i]], top[i, :k[i]])
        assert np.all(draft[i, k[i]:] != top[i, k[i]:])
        assert draft[i].min() >= 0 and draft[i].max() < V
