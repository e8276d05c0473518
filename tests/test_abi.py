"""The C-ABI library loads and exports every symbol include/lod.h declares, and
its host-side validation rejects bad arguments with the documented codes.
No call here reaches a GPU: every case fails validation before any launch,
or only sizes buffers."""
import ctypes
import os
import re

import pytest

import hierarchical_long_context_b200 as lod
from hierarchical_long_context_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    return _lib.load()


def _declared():
    src = open(os.path.join(ROOT, "include", "lod.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lod_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert set(declared) == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name
    assert L.lod_version() >= 100


def P(**kw):
    base = dict(B=2, Hq=16, Hkv=2, d=128, Tmax=4096)
    base.update(kw)
    return lod.Params(**base)


def _sizes(p):
    sizes = (ctypes.c_size_t * len(_lib.INDEX_FIELDS))()
    rc = _lib.load().lod_index_sizes(ctypes.byref(p.c()), sizes)
    return rc, list(sizes)


def test_index_sizes_match_the_documented_layout():
    p = P()
    rc, s = _sizes(p)
    assert rc == 0
    Cmax, k, Pp = 4096 // 256, 4, 256 // 16 + 4
    u = 2 * 2
    assert s == [u * Cmax * k * 128 * 2] * 2 + [u * Cmax * k * 4] + [u * Cmax * Pp * 128 * 2] * 2 + \
        [u * Cmax * Pp * 4, u * Cmax * Pp * 2, u * Cmax * (k + 1) * 2, u * Cmax * 256 * 2] + \
        [u * Cmax * 256 * 128 * 2] * 2 + [u * Cmax * k * 4] + [0] * 4


def test_int4_index_sizes_replace_the_member_copies():
    p = P(kv_bits=4)
    rc, s = _sizes(p)
    assert rc == 0
    Cmax, Pp, u = 4096 // 256, 256 // 16 + 4, 2 * 2
    assert s[9] == s[10] == 0
    assert s[12] == s[13] == u * Cmax * 256 * 128 // 2
    assert s[14] == s[15] == u * Cmax * Pp * 128 * 2 * 4


@pytest.mark.parametrize("kw", [dict(kv_bits=8), dict(kv_bits=4, top_pages=0)])
def test_unsupported_int4_settings(kw):
    rc, _ = _sizes(P(**kw))
    assert rc == _lib.LOD_EUNSUPPORTED


@pytest.mark.parametrize("kw, code", [
    (dict(d=96), _lib.LOD_EUNSUPPORTED),
    (dict(Hq=12, Hkv=8), _lib.LOD_EINVAL),
    (dict(Hq=48, Hkv=8), _lib.LOD_EUNSUPPORTED),     # g = 6 is not a power of two
    (dict(Hq=128, Hkv=8), _lib.LOD_EUNSUPPORTED),    # g = 16
    (dict(Hq=16, Hkv=1, d=64), _lib.LOD_EUNSUPPORTED),
    (dict(window=300), _lib.LOD_EINVAL),
    (dict(window=0), _lib.LOD_EINVAL),
    (dict(sinks=256), _lib.LOD_EINVAL),
    (dict(Tmax=1000), _lib.LOD_EINVAL),
    (dict(clusters=17), _lib.LOD_EUNSUPPORTED),
    (dict(top_groups=0), _lib.LOD_EUNSUPPORTED),
    (dict(top_pages=5), _lib.LOD_EUNSUPPORTED),
    (dict(chunk=128), _lib.LOD_EUNSUPPORTED),
    (dict(page=8), _lib.LOD_EUNSUPPORTED),
    (dict(B=0), _lib.LOD_EINVAL),
])
def test_bad_params_are_rejected(kw, code):
    rc, _ = _sizes(P(**kw))
    assert rc == code
    assert _lib.load().lod_last_error().decode()


def test_workspace_sizes_grow_with_the_problem():
    small = lod.workspace_bytes(P(), lod.LOD_OP_DECODE)
    big = lod.workspace_bytes(P(Tmax=131072), lod.LOD_OP_DECODE)
    assert big > small > 256
    assert lod.workspace_bytes(P(), lod.LOD_OP_BUILD) == 256
    assert lod.workspace_bytes(P(), lod.LOD_OP_PREFILL) > 256
    n = ctypes.c_size_t()
    assert _lib.load().lod_workspace_bytes(ctypes.byref(P().c()), 7, ctypes.byref(n)) == _lib.LOD_EINVAL


def test_null_and_misaligned_pointers_fail_before_any_launch():
    L = _lib.load()
    p = P().c()
    ix = _lib.lod_index()
    st = (ctypes.c_int64 * 3)(2 * 4096 * 128, 4096 * 128, 128)
    # NULL K/V
    rc = L.lod_build_index(ctypes.byref(p), None, None, st, 0, 1, ctypes.byref(ix), None, 0, None)
    assert rc == _lib.LOD_EINVAL
    # NULL index fields (fake, never dereferenced: validation stops first)
    fake = ctypes.c_void_p(1 << 20)
    rc = L.lod_build_index(ctypes.byref(p), fake, fake, st, 0, 1, ctypes.byref(ix), fake, 256, None)
    assert rc == _lib.LOD_EINVAL and b"index" in L.lod_last_error()
    # misaligned K
    rc = L.lod_build_index(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 2), fake, st, 0, 1,
                           ctypes.byref(ix), fake, 256, None)
    assert rc == _lib.LOD_EINVAL and b"aligned" in L.lod_last_error()
    # stride not a multiple of 16 bytes
    bad = (ctypes.c_int64 * 3)(2 * 4096 * 128, 4096 * 128, 129)
    rc = L.lod_build_index(ctypes.byref(p), fake, fake, bad, 0, 1, ctypes.byref(ix), fake, 256, None)
    assert rc == _lib.LOD_EINVAL
    # chunk range beyond Tmax (index pointers present, fake)
    full = _lib.lod_index(*([1 << 20] * len(_lib.INDEX_FIELDS)))
    rc = L.lod_build_index(ctypes.byref(p), fake, fake, st, 0, 17, ctypes.byref(full), fake, 256, None)
    assert rc == _lib.LOD_EINVAL and b"chunk range" in L.lod_last_error()
    rc = L.lod_build_index(ctypes.byref(p), fake, fake, st, 3, 3, ctypes.byref(full), fake, 256, None)
    assert rc == _lib.LOD_EINVAL
    # workspace too small for decode
    rc = L.lod_decode(ctypes.byref(p), fake, fake, fake, st, fake, ctypes.byref(full), fake, None, None,
                      None, fake, 256, None)
    assert rc == _lib.LOD_EINVAL and b"workspace" in L.lod_last_error()
    # prefill query range not chunk aligned
    rc = L.lod_prefill(ctypes.byref(p), fake, 100, 256, fake, fake, st, ctypes.byref(full), fake, None,
                       None, None, fake, 1 << 30, None)
    assert rc == _lib.LOD_EINVAL and b"query range" in L.lod_last_error()


def test_head_shard_must_lie_inside_the_model():
    sizes = (ctypes.c_size_t * len(_lib.INDEX_FIELDS))()
    for hs, rc in (((4 << 16) | 2, 0), ((4 << 16) | 3, _lib.LOD_EINVAL), ((1 << 16) | 0, _lib.LOD_EINVAL)):
        p = P(head_shard=hs).c()
        assert _lib.load().lod_index_sizes(ctypes.byref(p), sizes) == rc, hs


def test_struct_layout_matches_the_header():
    # offsets of the 64-bit members fixed by the header's field order
    assert _lib.lod_params.seed.offset == 56
    assert _lib.lod_params.scale.offset == 64
    assert _lib.lod_params.Tmax.offset == 72
    assert ctypes.sizeof(_lib.lod_params) == 80
    assert _lib.lod_params.kv_bits.offset == 52
    assert ctypes.sizeof(_lib.lod_index) == 8 * 16
