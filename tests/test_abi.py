"""The C-ABI library loads and exports every entry point include/ds4moe.h declares (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ds4moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ds4moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def libpath():
    from bit_quantized_moe_softmax_b200 import build

    return build.build()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("ds4moe_create", "ds4moe_pack_q2k", "ds4moe_pack_iq2xxs", "ds4moe_forward"):
        assert n in names


def test_library_exports_every_declared_symbol(libpath):
    lib = ctypes.CDLL(libpath)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", libpath], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (ds4moe_\w+)", out))
    assert set(_declared()) <= exported


def test_binding_names_match_header(libpath):
    import bit_quantized_moe_softmax_b200 as m

    assert set(m.EXPORTS) == set(_declared())
    for name in _declared():
        assert callable(getattr(m, name)), name


def test_last_error_without_gpu(libpath):
    import bit_quantized_moe_softmax_b200 as m

    assert isinstance(m.ds4moe_last_error(), str)


def _declarations():
    """{name: parameter count} for every function the header declares."""
    src = open(os.path.join(ROOT, "include", "ds4moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for name, params in re.findall(r"\b(ds4moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src):
        p = " ".join(params.split())
        out[name] = 0 if p in ("", "void") else p.count(",") + 1
    return out


def test_binding_signatures_match_header(libpath):
    """Every ctypes signature has as many arguments as the C declaration, and
    the shape struct's fields come in the header's order."""
    import bit_quantized_moe_softmax_b200 as m

    decl = _declarations()
    assert set(decl) == set(_declared())
    L = m.lib()
    for name, count in decl.items():
        assert len(getattr(L, name).argtypes) == count, (name, count)
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "ds4moe.h")).read(), flags=re.S)
    body = re.search(r"typedef struct\s*\{(.*?)\}\s*ds4moe_shape\s*;", src, flags=re.S).group(1)
    fields = re.findall(r"\b(\w+)\s*;", body)
    assert fields == [f for f, _ in m.ds4moe_shape._fields_]
    assert all(t is ctypes.c_int32 for _, t in m.ds4moe_shape._fields_)
    assert "int32_t" in body and not re.search(r"\b(int64_t|size_t|float|double)\b", body)


def test_q4_shape_rules_without_gpu(libpath):
    """Shape checks come before any CUDA call: 4-bit layers need inter a
    multiple of 256; other bit widths are refused."""
    import bit_quantized_moe_softmax_b200 as m

    for kw, why in ((dict(inter=128), "inter"), (dict(expert_bits=3), "bits"), (dict(expert_bits=1), "bits1")):
        args = dict(inter=256, max_tokens=8, decode_max=0, expert_bits=4)
        args.update(kw)
        with pytest.raises(m.Ds4MoeError) as ei:
            m.ds4moe_create(256, args["inter"], 8, 2, args["max_tokens"], decode_max=args["decode_max"],
                            expert_bits=args["expert_bits"])
        assert ei.value.status == -3, why
