"""Host-side checks of the C ABI that need no GPU: the library loads, exports every
symbol the header declares, and rejects bad configurations before touching CUDA."""
import ctypes as C
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from hybrid_deltanet_attention_b200 import build, _abi
    build.build()
    return _abi.load_library()


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "mk.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z_]+)\s*\(", txt)))


def test_header_and_binding_agree():
    from hybrid_deltanet_attention_b200 import _abi
    assert declared_symbols() == sorted(_abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_struct_sizes_match_c(lib, tmp_path):
    from hybrid_deltanet_attention_b200 import _abi
    src = tmp_path / "s.c"
    src.write_text('#include <stdio.h>\n#include "mk.h"\nint main(){printf("%zu %zu %zu", sizeof(mk_config),'
                   ' sizeof(mk_tensor), sizeof(mk_sizes));}\n')
    exe = tmp_path / "s"
    import subprocess
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)])
    out = subprocess.check_output([str(exe)]).decode().split()
    assert [int(x) for x in out] == [C.sizeof(_abi.MkConfig), C.sizeof(_abi.MkTensor), C.sizeof(_abi.MkSizes)]


def _cfg(**kw):
    from hybrid_deltanet_attention_b200 import make_config
    return make_config(synth.with_changes(synth.TINY, **kw), max_ctx=64)


@pytest.mark.parametrize("kw,frag", [
    (dict(pattern="DDXA"), "pattern"),
    (dict(n_layers=3), "pattern length"),
    (dict(hidden=100), "hidden"),
    (dict(dn_dk=48), "DeltaNet"),
    (dict(at_q_heads=3, at_kv_heads=2), "Hq"),
    (dict(at_head_dim=96), "at_head_dim"),
    (dict(conv_width=1), "conv_width"),
])
def test_bad_config_rejected_without_cuda(lib, kw, frag):
    from hybrid_deltanet_attention_b200 import _abi
    c = _cfg(**kw)
    sz = _abi.MkSizes()
    rc = lib.mk_query_sizes(C.byref(c), C.byref(sz))
    assert rc == _abi.MK_ERR_ARG
    assert frag in lib.mk_last_error().decode()


def test_null_arguments_rejected(lib):
    from hybrid_deltanet_attention_b200 import _abi
    assert lib.mk_query_sizes(None, None) == _abi.MK_ERR_ARG
    assert lib.mk_decode_step(None, None, None, None, None) == _abi.MK_ERR_ARG
    assert lib.mk_prefill(None, None, 0, None, None, None) == _abi.MK_ERR_ARG
    assert lib.mk_verify_drafts(None, None, 1, None, None, None, None) == _abi.MK_ERR_ARG
    assert lib.mk_verify_drafts_sampled(None, None, 1, 1.0, None, None, None, None, None) == _abi.MK_ERR_ARG
    assert lib.mk_generate(None, None, 0, None, 0, None) == _abi.MK_ERR_ARG
    assert lib.mk_launch_count(None) == 0
    lib.mk_free(None)


def test_no_cpu_fallback_when_library_missing(tmp_path):
    from hybrid_deltanet_attention_b200 import _abi
    saved = _abi._lib
    _abi._lib = None
    try:
        with pytest.raises(ImportError):
            _abi.load_library(str(tmp_path / "libmk.so"))
    finally:
        _abi._lib = saved
