"""ctypes view of liblod.so: the structs and prototypes of include/lod.h.

Argument marshalling only; every step of the method runs in the CUDA library.
The library must have been built (hierarchical_long_context_b200.build); there
is no fallback, and loading fails loudly when it is missing.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblod.so")

LOD_OK, LOD_EINVAL, LOD_EUNSUPPORTED, LOD_ECUDA, LOD_EDEVICE = 0, -1, -2, -3, -4
LOD_DTYPE_F32, LOD_DTYPE_BF16 = 0, 1
LOD_OP_BUILD, LOD_OP_DECODE, LOD_OP_PREFILL = 0, 1, 2
LOD_ST_BAD_SEQLEN, LOD_ST_BAD_PAGE, LOD_ST_BAD_MEMBER, LOD_ST_BAD_COUNT = 1, 2, 4, 8

# Every symbol include/lod.h declares.
EXPORTS = ("lod_version", "lod_last_error", "lod_index_sizes", "lod_workspace_bytes",
           "lod_build_index", "lod_build_ready", "lod_append_kv", "lod_decode", "lod_prefill", "lod_get_status",
           "lod_decode_noalloc")
NOALLOC_SCRATCH_BYTES = 8 << 20


class lod_params(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
        ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("page", ctypes.c_int32), ("clusters", ctypes.c_int32), ("kmeans_iters", ctypes.c_int32),
        ("top_groups", ctypes.c_int32), ("top_pages", ctypes.c_int32), ("window", ctypes.c_int32),
        ("sinks", ctypes.c_int32), ("kv_bits", ctypes.c_int32), ("seed", ctypes.c_uint64),
        ("scale", ctypes.c_float), ("head_shard", ctypes.c_int32), ("Tmax", ctypes.c_int64),
    ]


class lod_index(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("gK", "gV", "gCnt", "pK", "pV", "pCnt", "pBeg", "gPage", "perm", "mK", "mV", "gMeta",
                 "qK", "qV", "qKs", "qVs")]


INDEX_FIELDS = [f for f, _ in lod_index._fields_]

_P = ctypes.POINTER
_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_lib = None


class LodError(RuntimeError):
    def __init__(self, fn, code, msg):
        super().__init__("%s failed (%d): %s" % (fn, code, msg))
        self.code = code


def load():
    """Load liblod.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "liblod.so is not built (%s); run `python -m hierarchical_long_context_b200.build`"
            % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    lib.lod_version.restype = ctypes.c_int32
    lib.lod_version.argtypes = []
    lib.lod_last_error.restype = ctypes.c_char_p
    lib.lod_last_error.argtypes = []
    lib.lod_index_sizes.restype = ctypes.c_int32
    lib.lod_index_sizes.argtypes = [_P(lod_params), _P(ctypes.c_size_t)]
    lib.lod_workspace_bytes.restype = ctypes.c_int32
    lib.lod_workspace_bytes.argtypes = [_P(lod_params), ctypes.c_int32, _P(ctypes.c_size_t)]
    lib.lod_build_index.restype = ctypes.c_int32
    lib.lod_build_index.argtypes = [_P(lod_params), _vp, _vp, _P(_i64), _i64, _i64, _P(lod_index),
                                    _vp, ctypes.c_size_t, _vp]
    lib.lod_append_kv.restype = ctypes.c_int32
    lib.lod_append_kv.argtypes = [_P(lod_params), _vp, _vp, _P(_i64), _vp, _vp, _vp, _vp]
    lib.lod_build_ready.restype = ctypes.c_int32
    lib.lod_build_ready.argtypes = [_P(lod_params), _vp, _vp, _P(_i64), _vp, _P(lod_index), _vp,
                                    ctypes.c_size_t, _vp]
    lib.lod_decode.restype = ctypes.c_int32
    lib.lod_decode.argtypes = [_P(lod_params), _vp, _vp, _vp, _P(_i64), _vp, _P(lod_index), _vp, _vp,
                               _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.lod_prefill.restype = ctypes.c_int32
    lib.lod_prefill.argtypes = [_P(lod_params), _vp, _i64, _i64, _vp, _vp, _P(_i64), _P(lod_index),
                                _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    lib.lod_decode_noalloc.restype = ctypes.c_int32
    lib.lod_decode_noalloc.argtypes = [_P(lod_params), _vp, _vp, _vp, _P(_i64), _vp, _P(lod_index), _vp,
                                       _vp, _vp, _vp, _vp, _vp]
    lib.lod_get_status.restype = ctypes.c_int32
    lib.lod_get_status.argtypes = [_vp, _vp, _P(ctypes.c_uint32)]
    _lib = lib
    return lib


def check(fn: str, rc: int) -> int:
    if rc != LOD_OK:
        raise LodError(fn, rc, load().lod_last_error().decode())
    return rc
