"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad descriptors and handles before touching a
device."""
import ctypes
import os
import re

import pytest

from selective_state_space_forward_b200 import ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_forward_b200.build import build
    build()
    return ssd.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_the_binding_lists():
    assert _declared_functions() == sorted(ssd.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def _declared_param_counts():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(ssd_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_signatures_match_the_header(lib):
    counts = _declared_param_counts()
    assert sorted(counts) == sorted(ssd.EXPORTS)
    for name, n in counts.items():
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None and len(argtypes) == n, (name, n, argtypes)


def test_status_strings(lib):
    for code, name in ssd.STATUS_NAMES.items():
        assert lib.ssd_status_string(code).decode() == name
    assert lib.ssd_status_string(99).decode() == "SSD_ERR_UNKNOWN"


def _desc(**kw):
    base = dict(nheads=4, headdim=16, dstate=16, ngroups=1, dconv=4, chunk=64, act_dtype=1,
                a_mode=0, bc_norm=0, max_batch=1, max_seqlen=64, path=0)
    base.update(kw)
    return ssd.Desc(**base)


@pytest.mark.parametrize("kw,status,word", [
    (dict(nheads=0), 1, "nheads"),
    (dict(headdim=12), 2, "headdim"),
    (dict(headdim=256), 2, "headdim"),
    (dict(dstate=4), 2, "dstate"),
    (dict(ngroups=3), 1, "ngroups"),
    (dict(dconv=3), 2, "dconv"),
    (dict(chunk=128), 2, "chunk"),
    (dict(act_dtype=7), 1, "act_dtype"),
    (dict(a_mode=2), 1, "a_mode"),
    (dict(bc_norm=2), 1, "bc_norm"),
    (dict(max_batch=0), 1, "max_batch"),
    (dict(path=9), 1, "path"),
    (dict(validate_finite=2), 1, "validate_finite"),
    (dict(path=1, act_dtype=0), 2, "fused"),
    (dict(path=1, headdim=32), 2, "fused"),
])
def test_bad_descriptor_is_refused_by_name(lib, kw, status, word):
    h = ctypes.c_void_p()
    st = lib.ssd_create(ctypes.byref(_desc(**kw)), ctypes.byref(h))
    assert st == status
    assert word in lib.ssd_last_error().decode()
    assert not h.value


def test_null_handle_is_refused(lib):
    st = lib.ssd_forward(None, 1, 1, *([None] * 15))
    assert st == 1 and "handle" in lib.ssd_last_error().decode()
    st = lib.ssd_step(None, 1, *([None] * 13))
    assert st == 1
    assert st == 1
    assert lib.ssd_check(None, None) == 1
    assert lib.ssd_get_path(None) == -1
    assert lib.ssd_state_bytes(None, 1) == 0
    lib.ssd_destroy(None)   # no-op


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        ssd.load_library(str(tmp_path / "libssd.so"))
