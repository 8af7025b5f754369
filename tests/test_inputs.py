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


@pytest.mark.parametrize("dims", [gen.TINY, gen.ModelDims(n_layers=2, hidden=256, n_q_heads=8, n_kv_heads=1,
                                                           head_dim=128, inter=192, vocab=512, dtype="bf16")])
def test_uploaded_layout_matches_the_abi_and_the_oracle_names(dims):
    """The uploader stacks each layer's matrices as the C ABI documents
    (wqkv rows: the Hq query heads, then the Hkv key heads, then the Hkv
    value heads, D rows each; wo, wgate, wup, wdown [out, in]) from exactly
    the draws the oracle uses under its own names; caches are K [layers,
    batch, Hkv, Lmax, D] and V transposed [layers, batch, Hkv, D, Lmax]."""
    import oracle as O
    from dvlm_gen.device import DeviceModel, as_f64, kv_buffers
    dm = DeviceModel(dims, 3, device="cpu")
    w = O.weights_from_generator(gen, dims, 3)
    qd, kd = dims.n_q_heads * dims.head_dim, dims.n_kv_heads * dims.head_dim
    for l in range(dims.n_layers):
        qkv = as_f64(dm.wqkv[l])
        assert np.array_equal(qkv[:qd], w[f"{l}.wq"])
        assert np.array_equal(qkv[qd:qd + kd], w[f"{l}.wk"])
        assert np.array_equal(qkv[qd + kd:], w[f"{l}.wv"])
        for name, t in (("wo", dm.wo), ("wg", dm.wgate), ("wu", dm.wup), ("wd", dm.wdown)):
            assert np.array_equal(as_f64(t[l]), w[f"{l}.{name}"]), name
    assert np.array_equal(as_f64(dm.embed), w["embed"]) and np.array_equal(as_f64(dm.lm_head), w["lm_head"])
    k, v = kv_buffers(dims, 40, device="cpu", n_batch=2)
    assert k.shape == (dims.n_layers, 2, dims.n_kv_heads, 40, dims.head_dim)
    assert v.shape == (dims.n_layers, 2, dims.n_kv_heads, dims.head_dim, 40)
    m = dm.c_model()
    assert (m.n_layers, m.hidden, m.n_q_heads, m.n_kv_heads, m.head_dim, m.inter, m.vocab, m.mask_id) == \
        (dims.n_layers, dims.hidden, dims.n_q_heads, dims.n_kv_heads, dims.head_dim, dims.inter, dims.vocab,
         dims.vocab - 1)
    assert m.wqkv == dm.wqkv.data_ptr() and m.lm_head == dm.lm_head.data_ptr()
