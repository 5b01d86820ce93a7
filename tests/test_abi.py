"""Host-side tests of the C ABI (no GPU): the library loads, exports every entry
point include/dz.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

from causal_video_diffusion_rope_b200 import build, dz

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return dz.load()


def _declared_functions():
    names = set()
    include = os.path.join(ROOT, "include")
    for f in os.listdir(include):
        if not f.endswith(".h"):
            continue
        text = open(os.path.join(include, f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(dz_[A-Za-z0-9_]+)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared_functions()
    assert {"dz_attn_create", "dz_chunk_attn_forward", "dz_rope3d", "dz_kvcache_append",
            "dz_kvcache_replace"} <= declared
    for name in declared:
        assert hasattr(lib, name), f"libdz.so does not export {name}"
    assert set(dz.EXPORTS) <= declared


def test_status_strings(lib):
    assert dz.status_string(0) == "ok"
    for s in range(1, 9):
        assert dz.status_string(s) not in ("ok", "unknown status")
    assert dz.status_string(99) == "unknown status"


def test_create_rejects_bad_descriptors(lib):
    h = ctypes.c_void_p()
    assert lib.dz_attn_create(ctypes.byref(h), None) == dz.DZ_ERR_INVALID_ARG
    d = dz.make_desc()
    d.head_dim = 64
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(d)) == dz.DZ_ERR_SHAPE
    d = dz.make_desc(pairs=(22, 21, 20))
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(d)) == dz.DZ_ERR_SHAPE
    d = dz.make_desc(num_heads=0)
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(d)) == dz.DZ_ERR_SHAPE
    d = dz.make_desc(max_q_tokens=2048 * 256 + 1)
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(d)) == dz.DZ_ERR_CAPACITY
    d = dz.make_desc(rope_base=1.0)
    assert lib.dz_attn_create(ctypes.byref(h), ctypes.byref(d)) == dz.DZ_ERR_SHAPE


def test_calls_reject_null_handle(lib):
    lay = dz.make_layout(dz.DZ_MODE_DECODE, 1, 2, 11, 20, 24, 4)
    cache = dz.make_cache(16, 16, 1, 10, 0, 464)
    assert lib.dz_chunk_attn_forward(None, 16, 16, 16, None, ctypes.byref(lay), 16, None) == \
        dz.DZ_ERR_INVALID_ARG
    assert lib.dz_rope3d(None, 16, 16, 1, 1, ctypes.byref(lay), 0, None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_kvcache_append(None, ctypes.byref(cache), 16, 16, None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_kvcache_replace(None, ctypes.byref(cache), 0, 16, 16, None) == \
        dz.DZ_ERR_INVALID_ARG
    # a NULL handle asks for the allocation-free calls' status word: without a device the
    # stream synchronisation fails, on a device with no such call yet it is clear
    assert lib.dz_attn_sync_status(None, None) in (dz.DZ_OK, dz.DZ_ERR_CUDA)
    assert lib.dz_attn_destroy(None) == dz.DZ_ERR_INVALID_ARG
    pre = dz.make_layout(dz.DZ_MODE_PREFILL, 1, 1, 4, 4, 4, 2)
    assert lib.dz_qkv_rope(None, 16, 16, 1, 20, 128, ctypes.byref(pre), 0, 16, 16, 16, None,
                           None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_chunk_attn_forward_lse(None, 16, 16, 16, ctypes.byref(pre), 16, 16, None) == \
        dz.DZ_ERR_INVALID_ARG
    assert lib.dz_chunk_attn_backward(None, 16, 16, 16, 16, 16, 16, ctypes.byref(pre), 16, 16,
                                      16, None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_chunk_attn_forward_e4m3(None, 16, 16, 16, None, ctypes.byref(lay), 64.0, 16.0,
                                          16, None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_quantize_e4m3(None, 16, 16, 128, 1.0, None) == dz.DZ_ERR_INVALID_ARG
    assert lib.dz_rope3d_e4m3(None, 16, 32, 1, 1, ctypes.byref(lay), 0, 1.0, None) == \
        dz.DZ_ERR_INVALID_ARG
    # a null layout or output pointer is rejected before any handle lookup
    assert lib.dz_chunk_attn_forward_lse(None, 16, 16, 16, None, 16, 16, None) == \
        dz.DZ_ERR_INVALID_ARG
    assert lib.dz_chunk_attn_backward(None, 16, 16, 16, 16, 16, None, ctypes.byref(pre), 16, 16,
                                      16, None) == dz.DZ_ERR_INVALID_ARG


def test_python_binding_raises(lib):
    with pytest.raises(dz.DzError) as e:
        d = dz.make_desc()
        d.head_dim = 96
        dz.dz_attn_create(d)
    assert e.value.status == dz.DZ_ERR_SHAPE


def test_binding_has_same_names_as_header():
    declared = _declared_functions()
    for name in declared:
        assert hasattr(dz, name), f"binding lacks {name}"


def test_struct_layouts_match_the_header(tmp_path):
    """Size and field offsets of the public structs as a C compiler lays them out from
    include/dz.h, against the binding's ctypes definitions."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    structs = {"dz_attn_desc": dz.dz_attn_desc, "dz_chunk_layout": dz.dz_chunk_layout,
               "dz_kvcache": dz.dz_kvcache}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "dz.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ['  printf("DZ_MODE_ROTATED %d\\n", DZ_MODE_ROTATED);', "  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n"):
        if line:
            *key, value = line.split()
            got[" ".join(key)] = int(value)
    for name, cls in structs.items():
        assert got[f"{name} size"] == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert got[f"{name} {field}"] == getattr(cls, field).offset, (name, field)
    assert got["DZ_MODE_ROTATED"] == dz.DZ_MODE_ROTATED
