"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/dvlm.h declares, validates arguments on the host (returning a
status before any launch) and lays its structs out as the header does."""
import ctypes
import os
import subprocess


import block_diffusion_vlm_b200 as dv
from block_diffusion_vlm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, SHAPE, UNSUPPORTED, OVERFLOW, TIMEOUT, CUDA, WORKSPACE, BOUNDS = range(9)


def test_library_exports_every_declared_symbol(dvlm_lib):
    names = dv.declared_symbols()
    assert len(names) >= 19
    for n in names:
        assert hasattr(dvlm_lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) == {e for e in exported if e.startswith("dvlm_")}


def test_status_strings_and_version(dvlm_lib):
    assert dv.status_string(0) == "ok"
    assert "timed out" in dv.status_string(TIMEOUT)
    assert dv.status_string(999) == "unknown status"
    assert dvlm_lib.dvlm_version() == 100


def test_struct_layouts_match_header(tmp_path):
    src = tmp_path / "sz.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "dvlm.h"\n'
                   'int main(){printf("%zu %zu %zu %zu %zu\\n", sizeof(dvlm_model), sizeof(dvlm_decode_cfg),'
                   ' sizeof(dvlm_stats), offsetof(dvlm_model, lm_head), offsetof(dvlm_stats, accept_hist));}\n')
    exe = tmp_path / "sz"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()]
    want = [ctypes.sizeof(dv.Model), ctypes.sizeof(dv.DecodeCfg), ctypes.sizeof(dv.Stats),
            dv.Model.lm_head.offset, dv.Stats.accept_hist.offset]
    assert got == want


def _attn(**kw):
    a = dict(q=16, out=16, k=16, v=16, nb=1, n_rows=16, n_clean=0, L=64, Lmax=128, Hq=16, Hkv=2, D=128,
             scale=0.088, dt=0)
    a.update(kw)
    return dv.lib().dvlm_block_attn(a["q"], a["out"], a["k"], a["v"], a["nb"], a["n_rows"], a["n_clean"], a["L"],
                                    a["Lmax"], a["Hq"], a["Hkv"], a["D"], a["scale"], a["dt"], None, None)


def test_attention_host_validation(dvlm_lib):
    assert _attn(q=None) == INVALID
    assert _attn(dt=7) == INVALID
    assert _attn(scale=float("inf")) == INVALID
    assert _attn(n_clean=17) == SHAPE
    assert _attn(Hq=15) == SHAPE
    assert _attn(L=120) == OVERFLOW
    assert _attn(D=64) == UNSUPPORTED
    assert _attn(Hq=8) == UNSUPPORTED
    assert _attn(Lmax=130, L=64) == SHAPE
    assert _attn(q=18) == INVALID      # misaligned for the TMA path


def _lm(**kw):
    a = dict(h=16, w=16, R=16, H=2048, V=151936, dt=0, norm=0, eps=1e-6, masked=None, tokens=None, thr=0.9,
             aid=None, aconf=None, cert=None, ws=16, wsb=1 << 40)
    a.update(kw)
    return dv.lib().dvlm_lmhead_conf_commit(a["h"], a["w"], a["R"], a["H"], a["V"], a["dt"], a["norm"], a["eps"],
                                            a["masked"], a["tokens"], a["thr"], None, None, None, None, a["aid"],
                                            a["aconf"], a["cert"], a["ws"], a["wsb"], None, None)


def test_lmhead_host_validation(dvlm_lib):
    assert _lm(h=None) == INVALID
    assert _lm(R=0) == SHAPE and _lm(R=129) == SHAPE
    assert _lm(tokens=64) == INVALID                 # tokens need masked
    assert _lm(aid=64) == INVALID                    # certificate is all-or-none
    assert _lm(thr=float("nan")) == INVALID
    assert _lm(ws=None) == WORKSPACE
    assert _lm(wsb=100) == WORKSPACE
    assert _lm(H=100) == UNSUPPORTED
    assert _lm(h=24) == INVALID
    assert dv.lmhead_workspace_size(0, 10, 10, 0) == 0
    assert dv.lmhead_workspace_size(16, 151936, 2048, 0) > 0


def test_spec_host_validation(dvlm_lib):
    L = dv.lib()
    f = L.dvlm_spec_verify_accept
    assert f(None, 16, None, 1, 16, 100, 16, None, 0, None, None, 0, 0, 0, 0, None, 0, None, None) == INVALID
    assert f(None, None, 16, 1, 16, 100, 16, None, 0, None, None, 0, 0, 0, 0, None, 0, None, None) == INVALID
    assert f(None, 16, 16, 1, 16, 100, None, None, 0, None, None, 0, 0, 0, 0, None, 0, None, None) == INVALID
    assert f(None, 16, 16, 1, 65, 100, 16, None, 0, None, None, 0, 0, 0, 0, None, 0, None, None) == SHAPE
    assert f(16, None, 16, 1, 16, 100, 16, None, 0, None, None, 0, 0, 0, 0, None, 0, None, None) == WORKSPACE
    assert f(None, 16, 16, 1, 16, 100, 16, None, 1, None, None, 0, 0, 0, 0, None, 0, None, None) == INVALID


def test_topk_host_validation(dvlm_lib):
    f = dv.lib().dvlm_topk_commit
    assert f(None, 16, 16, 16, 4, 1, None, None, None, None) == INVALID
    assert f(16, 16, 16, None, 4, 1, None, None, None, None) == INVALID
    assert f(16, 16, 16, 16, 0, 1, None, None, None, None) == SHAPE
    assert f(16, 16, 16, 16, 129, 1, None, None, None, None) == SHAPE
    assert f(16, 16, 16, 16, 4, -1, None, None, None, None) == SHAPE
    g = dv.lib().dvlm_divergence_first_commit
    assert g(16, 16, None, 16, 16, 4, 1, None, None, None, None) == INVALID
    assert g(16, 16, 16, 16, 16, 129, 1, None, None, None, None) == SHAPE
    assert g(16, 16, 16, 16, 16, 4, -2, None, None, None, None) == SHAPE


def _dims_model(**kw):
    import dvlm_gen as gen
    m = dv.make_model(gen.QWEN3B, embed=None, wqkv=None, wo=None, wgate=None, wup=None, wdown=None,
                      lm_head=None, dtype=0)
    for name in ("embed", "wqkv", "wo", "wgate", "wup", "wdown", "lm_head"):
        setattr(m, name, 4096)
    for k, v in kw.items():
        setattr(m, k, v)
    return m


def test_engine_host_validation(dvlm_lib):
    L = dv.lib()
    m = _dims_model()
    ws = dv.engine_workspace_size(m, 1600, 16, 1344)
    assert ws > 0
    assert dv.engine_workspace_size(_dims_model(n_kv_heads=3), 1600, 16, 1344) == 0
    assert dv.engine_workspace_size(_dims_model(mask_id=151936), 1600, 16, 1344) == 0
    assert dv.engine_workspace_size(m, 1600, 17, 1344) == 0
    h = ctypes.c_void_p()
    assert L.dvlm_engine_create(ctypes.byref(m), 4096, 4096, 1600, 16, 0, 4096, ws, None, None) == INVALID
    assert L.dvlm_engine_create(ctypes.byref(m), None, 4096, 1600, 16, 0, 4096, ws, None, ctypes.byref(h)) == INVALID
    assert L.dvlm_engine_create(ctypes.byref(_dims_model(head_dim=64)), 4096, 4096, 1600, 16, 0, 4096, ws, None,
                                ctypes.byref(h)) == UNSUPPORTED
    assert L.dvlm_engine_create(ctypes.byref(m), 4096, 4096, 1601, 16, 0, 4096, ws, None,
                                ctypes.byref(h)) == INVALID
    assert L.dvlm_engine_create(ctypes.byref(m), 4096, 4096, 1600, 16, 0, None, ws, None,
                                ctypes.byref(h)) == WORKSPACE
    assert L.dvlm_engine_destroy(None) == INVALID
    assert L.dvlm_prefill(None, None, 0, None, 0, None) == INVALID
    assert L.dvlm_decode_block(None, None, None, None, None, None) == INVALID
    assert L.dvlm_forward_text_only(None, 4096, None, 16, 32, None, None) == INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without the built library every entry point raises."""
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libdvlm.so"))
    import pytest
    with pytest.raises(RuntimeError, match="missing"):
        binding.lib()
    with pytest.raises(RuntimeError, match="missing"):
        dv.topk_commit(None, None, None, None, R=1, k=1)


def test_binding_declares_every_header_entry_point():
    """Every entry point of include/dvlm.h has a ctypes signature in the
    binding (so no call goes through ctypes' int defaults)."""
    import inspect
    import re
    src = inspect.getsource(binding._declare)
    assert set(re.findall(r'"(dvlm_\w+)"', src)) == set(dv.declared_symbols())
