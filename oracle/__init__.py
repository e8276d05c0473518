"""CPU oracle for Level-of-Detail attention: a ctypes wrapper over lod_oracle.c.

TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports this
package and this package never imports the CUDA library; they share nothing
but the seeded inputs that the tests hand to both.

Every function follows "Level of Detail Attention" (featherless.ai blog),
section "How It Works"; the C file's header lists the readings taken where
the page is silent.  The C code is single-threaded; the ctypes calls release
the GIL, so callers may run independent rows or sequences on a thread pool.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lod_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile lod_oracle.c into oracle/liboracle.so with gcc (plain -O2, no
    fast-math, so IEEE rounding of every operation is kept)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-Wall",
             "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Params(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int32), ("chunk", ctypes.c_int32), ("page", ctypes.c_int32),
        ("clusters", ctypes.c_int32), ("iters", ctypes.c_int32),
        ("top_groups", ctypes.c_int32), ("top_pages", ctypes.c_int32),
        ("window", ctypes.c_int32), ("sinks", ctypes.c_int32),
        ("store_bf16", ctypes.c_int32), ("seed", ctypes.c_uint64), ("scale", ctypes.c_double),
    ]


class RowStats(ctypes.Structure):
    _fields_ = [
        ("n_exact", ctypes.c_int64), ("n_coarse_groups", ctypes.c_int64),
        ("n_coarse_pages", ctypes.c_int64), ("covered", ctypes.c_int64),
        ("n_visible", ctypes.c_int64), ("weight_sum", ctypes.c_double),
        ("window_start", ctypes.c_double),
    ]


_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.orc_splitmix64.restype = ctypes.c_uint64
        lib.orc_splitmix64.argtypes = [ctypes.c_uint64]
        lib.orc_round_bf16.restype = ctypes.c_double
        lib.orc_round_bf16.argtypes = [ctypes.c_double]
        lib.orc_round_bf16_array.restype = None
        lib.orc_round_bf16_array.argtypes = [_f64p, _f64p, ctypes.c_int64]
        lib.orc_page_slots.restype = ctypes.c_int32
        lib.orc_page_slots.argtypes = [ctypes.POINTER(Params)]
        lib.orc_build_sequence.restype = ctypes.c_int
        lib.orc_build_sequence.argtypes = [
            ctypes.POINTER(Params), ctypes.c_uint64, _f32p, _f32p, ctypes.c_int64,
            _i32p, _f64p, _f64p, _i32p, _f64p, _f64p, _i32p, _i32p, _i32p, _i32p, _i32p,
            _f64p, _f64p, ctypes.c_void_p]
        lib.orc_attend_row.restype = ctypes.c_int
        lib.orc_attend_row.argtypes = [
            ctypes.POINTER(Params), _f32p, ctypes.c_int64, _f32p, _f32p, ctypes.c_int64,
            _f64p, _f64p, _i32p, _f64p, _f64p, _i32p, _i32p, _i32p, _i32p,
            ctypes.c_void_p, ctypes.c_void_p, _f64p, ctypes.POINTER(ctypes.c_double),
            _i32p, _i32p, ctypes.POINTER(RowStats)]
        lib.orc_quantize_pages.restype = ctypes.c_int
        lib.orc_quantize_pages.argtypes = [
            ctypes.POINTER(Params), _f32p, ctypes.c_int64, _i32p, _i32p, _i32p, _u8p, _f32p, _f32p]
        lib.orc_attend_row_q.restype = ctypes.c_int
        lib.orc_attend_row_q.argtypes = [
            ctypes.POINTER(Params), _f32p, ctypes.c_int64, _f32p, _f32p, ctypes.c_int64,
            _f64p, _f64p, _i32p, _f64p, _f64p, _i32p, _i32p, _i32p, _i32p,
            _u8p, _f32p, _f32p, _u8p, _f32p, _f32p,
            ctypes.c_void_p, ctypes.c_void_p, _f64p, ctypes.POINTER(ctypes.c_double),
            _i32p, _i32p, ctypes.POINTER(RowStats)]
        lib.orc_dense_row.restype = ctypes.c_int
        lib.orc_dense_row.argtypes = [
            ctypes.POINTER(Params), _f32p, ctypes.c_int64, _f32p, _f32p, _f64p,
            ctypes.POINTER(ctypes.c_double)]
        _lib = lib
    return _lib


@dataclass
class Config:
    """LoD parameters as the oracle sees them (one sequence, one KV head)."""
    d: int
    clusters: int = 4
    iters: int = 8
    top_groups: int = 8
    top_pages: int = 2
    window: int = 256
    sinks: int = 1
    store_bf16: bool = False
    seed: int = 0
    scale: float = 0.0
    chunk: int = 256
    page: int = 16

    def c(self) -> Params:
        return Params(self.d, self.chunk, self.page, self.clusters, self.iters, self.top_groups,
                      self.top_pages, self.window, self.sinks, int(self.store_bf16),
                      self.seed & (2**64 - 1), self.scale)

    @property
    def page_slots(self) -> int:
        return _load().orc_page_slots(ctypes.byref(self.c()))


def splitmix64(x: int) -> int:
    return int(_load().orc_splitmix64(x & (2**64 - 1)))


def round_bf16(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty_like(a)
    _load().orc_round_bf16_array(a.ravel(), out.ravel(), a.size)
    return out


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def build_sequence(cfg: Config, unit: int, K, V, nchunks: int, want_objective: bool = False) -> dict:
    """Index of one sequence: chunks [0, nchunks) of K, V ([T, d] arrays)."""
    lib = _load()
    K = _f32(K); V = _f32(V)
    assert K.shape == V.shape and K.shape[1] == cfg.d and K.shape[0] >= nchunks * cfg.chunk
    k, P, C, d = cfg.clusters, cfg.page_slots, cfg.chunk, cfg.d
    out = dict(
        assign=np.empty(nchunks * C, np.int32), gK=np.empty((nchunks * k, d)),
        gV=np.empty((nchunks * k, d)), gCnt=np.empty(nchunks * k, np.int32),
        pK=np.empty((nchunks * P, d)), pV=np.empty((nchunks * P, d)),
        pCnt=np.empty(nchunks * P, np.int32), pBeg=np.empty(nchunks * P, np.int32),
        gPage=np.empty(nchunks * (k + 1), np.int32), perm=np.empty(nchunks * C, np.int32),
        init_idx=np.empty(nchunks * k, np.int32), min_margin=np.empty(nchunks),
        key_margin=np.empty(nchunks * C))
    obj = np.empty(nchunks * cfg.iters) if want_objective else None
    rc = lib.orc_build_sequence(
        ctypes.byref(cfg.c()), unit, K, V, nchunks, out["assign"], out["gK"], out["gV"],
        out["gCnt"], out["pK"], out["pV"], out["pCnt"], out["pBeg"], out["gPage"], out["perm"],
        out["init_idx"], out["min_margin"], out["key_margin"],
        obj.ctypes.data_as(ctypes.c_void_p) if obj is not None else None)
    if rc != 0:
        raise ValueError("orc_build_sequence failed: %d" % rc)
    out["nchunks"] = nchunks
    if obj is not None:
        out["objective"] = obj.reshape(nchunks, cfg.iters)
    return out


def quantize_pages(cfg: Config, X, index: dict) -> dict:
    """Three-tier INT4 page quantiser (keys or values X, [T, d]) over the pages
    of `index`: code [nchunks*chunk, d] uint8 in member order, scale and low
    [nchunks*P, d] float32 per page slot and channel."""
    lib = _load()
    X = _f32(X)
    n, C, P, d = index["nchunks"], cfg.chunk, cfg.page_slots, cfg.d
    code = np.empty((n * C, d), np.uint8)
    scale = np.empty((n * P, d), np.float32)
    low = np.empty((n * P, d), np.float32)
    rc = lib.orc_quantize_pages(
        ctypes.byref(cfg.c()), X, n, np.ascontiguousarray(index["pCnt"], np.int32),
        np.ascontiguousarray(index["pBeg"], np.int32), np.ascontiguousarray(index["perm"], np.int32),
        code, scale, low)
    if rc != 0:
        raise ValueError("orc_quantize_pages failed: %d" % rc)
    return dict(code=code, scale=scale, low=low)


def attend_row(cfg: Config, q, t: int, K, V, index: dict, forced_groups=None, forced_pages=None,
               kq: dict = None, vq: dict = None):
    """LoD attention of one query at position t against one sequence's index.
    kq / vq (quantize_pages of K and V): the opened pages' members are read
    decompressed (three-tier INT4).  Returns (out[d] fp64, lse, sel_groups,
    sel_pages, stats dict)."""
    lib = _load()
    q = _f32(q); K = _f32(K); V = _f32(V)
    G, TP = cfg.top_groups, cfg.top_pages
    out = np.empty(cfg.d)
    lse = ctypes.c_double()
    sg = np.empty(G, np.int32)
    sp = np.empty(G * TP, np.int32)
    st = RowStats()
    fg = fp = None
    if forced_groups is not None:
        fg = np.ascontiguousarray(forced_groups, np.int32)
        assert fg.size == G
        fp = np.ascontiguousarray(forced_pages, np.int32)
        assert fp.size == G * TP
    qargs = []
    if kq is not None:
        qargs = [np.ascontiguousarray(kq["code"], np.uint8), _f32(kq["scale"]), _f32(kq["low"]),
                 np.ascontiguousarray(vq["code"], np.uint8), _f32(vq["scale"]), _f32(vq["low"])]
    fn = lib.orc_attend_row_q if kq is not None else lib.orc_attend_row
    rc = fn(
        ctypes.byref(cfg.c()), q, t, K, V, index["nchunks"],
        np.ascontiguousarray(index["gK"], np.float64), np.ascontiguousarray(index["gV"], np.float64),
        np.ascontiguousarray(index["gCnt"], np.int32), np.ascontiguousarray(index["pK"], np.float64),
        np.ascontiguousarray(index["pV"], np.float64), np.ascontiguousarray(index["pCnt"], np.int32),
        np.ascontiguousarray(index["pBeg"], np.int32), np.ascontiguousarray(index["gPage"], np.int32),
        np.ascontiguousarray(index["perm"], np.int32), *qargs,
        fg.ctypes.data_as(ctypes.c_void_p) if fg is not None else None,
        fp.ctypes.data_as(ctypes.c_void_p) if fp is not None else None,
        out, ctypes.byref(lse), sg, sp, ctypes.byref(st))
    if rc != 0:
        raise ValueError("orc_attend_row failed: %d" % rc)
    stats = {f: getattr(st, f) for f, _ in RowStats._fields_}
    return out, lse.value, sg, sp.reshape(G, TP), stats


def dense_row(cfg: Config, q, t: int, K, V):
    """Full softmax attention of one query at position t over [0, t] (fp64)."""
    lib = _load()
    out = np.empty(cfg.d)
    lse = ctypes.c_double()
    rc = lib.orc_dense_row(ctypes.byref(cfg.c()), _f32(q), t, _f32(K), _f32(V), out,
                           ctypes.byref(lse))
    if rc != 0:
        raise ValueError("orc_dense_row failed: %d" % rc)
    return out, lse.value
