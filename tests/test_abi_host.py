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
    assert lib.ssd_check(None, None) == 1
    assert lib.ssd_get_path(None) == -1
    assert lib.ssd_state_bytes(None, 1) == 0
    lib.ssd_destroy(None)   # no-op


def _s6(lib, batch=1, seqlen=8, d_inner=16, dstate=16, act_dtype=1, **ptrs):
    names = ("u", "delta", "delta_bias", "A_log", "B", "C", "D", "z", "init", "out", "fin")
    # distinct, aligned, never dereferenced: every case is refused before a launch
    p = {n: 0x10000 * (i + 1) for i, n in enumerate(names)}
    p.update(ptrs)
    return lib.ssd_s6_forward(batch, seqlen, d_inner, dstate, act_dtype,
                              *[p[n] for n in names], None)


@pytest.mark.parametrize("kw,status,word", [
    (dict(dstate=12), 2, "dstate"),
    (dict(act_dtype=5), 1, "act_dtype"),
    (dict(batch=-1), 1, "batch"),
    (dict(d_inner=0), 1, "d_inner"),
    (dict(init=0x10002), 3, "init_state"),
    (dict(u=None), 1, "u"),
    (dict(A_log=None), 1, "A_log"),
    (dict(out=0x10000), 1, "alias"),
])
def test_s6_bad_arguments_are_refused_by_name(lib, kw, status, word):
    assert _s6(lib, **kw) == status
    assert word in lib.ssd_last_error().decode()


def test_s6_empty_batch_is_a_no_op(lib):
    assert _s6(lib, batch=0) == 0


def test_noalloc_refuses_bad_descriptors(lib):
    st = lib.ssd_forward_noalloc(ctypes.byref(_desc(nheads=0)), 1, 1, *([None] * 16))
    assert st == 1 and "nheads" in lib.ssd_last_error().decode()
    st = lib.ssd_forward_noalloc(ctypes.byref(_desc(path=2)), 1, 1, *([None] * 16))
    assert st == 2 and "fused path only" in lib.ssd_last_error().decode()


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        ssd.load_library(str(tmp_path / "libssd.so"))
