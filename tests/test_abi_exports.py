"""The C-ABI library loads on a machine without a GPU and exports every
function that include/*.h declares (no compute call is made)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(polar_(?:attn|gdelta)_[A-Za-z0-9_]+)\s*\(",
                             src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("polar_attn_fwd", "polar_attn_decode_paged", "polar_attn_get_status",
                 "polar_gdelta_prefill", "polar_gdelta_step"):
        assert must in names


def _declaration(name):
    src = ""
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src += re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
    m = re.search(r"\b" + name + r"\s*\(([^)]*)\)\s*;", src)
    assert m, name
    return [" ".join(a.split()) for a in m.group(1).split(",")]


def test_prefill_entry_point_has_the_eight_argument_signature():
    """polar_attn_fwd(q, k, v, u, params, out, neff_out, stream): the prefill
    call with no workspace; the workspace form is polar_attn_fwd_ws."""
    args = _declaration("polar_attn_fwd")
    names = [a.replace("*", " ").split()[-1] for a in args]
    assert names == ["q", "k", "v", "u", "params", "out", "neff_out", "stream"], args
    ws = [a.replace("*", " ").split()[-1] for a in _declaration("polar_attn_fwd_ws")]
    assert ws == names[:-1] + ["workspace", "ws_bytes", "stream"], ws


def test_library_exports_every_declared_symbol():
    from polar_attention_b200 import native
    if not os.path.exists(native.LIB_PATH):
        from polar_attention_b200 import build
        build.build()
    lib = ctypes.CDLL(native.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, f"not exported: {missing}"
    assert set(native.EXPORTS) == set(declared_functions())


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    from polar_attention_b200 import native
    monkeypatch.setattr(native, "_lib", None)
    monkeypatch.setattr(native, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        native.lib()
