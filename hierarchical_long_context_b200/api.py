"""Python binding of the LoD attention library (torch tensors in, C ABI out).

Same names as the C entry points.  PyTorch provides device memory and the
current stream; the binding only checks shapes, allocates outputs and passes
pointers.  All arithmetic runs in liblod.so.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import check, load

_DT = {torch.float32: _lib.LOD_DTYPE_F32, torch.bfloat16: _lib.LOD_DTYPE_BF16}


@dataclass(frozen=True)
class Params:
    """Mirror of lod_params (include/lod.h)."""
    B: int
    Hq: int
    Hkv: int
    d: int
    Tmax: int
    dtype: torch.dtype = torch.bfloat16
    clusters: int = 4
    kmeans_iters: int = 8
    top_groups: int = 8
    top_pages: int = 2
    window: int = 512
    sinks: int = 4
    seed: int = 0
    scale: float = 0.0
    chunk: int = 256
    page: int = 16
    kv_bits: int = 0   # 4: three-tier INT4 (opened pages read from 4-bit codes)
    head_shard: int = 0  # (model KV heads << 16) | first KV head, for a head-sharded process

    def c(self) -> _lib.lod_params:
        return _lib.lod_params(
            _DT[self.dtype], self.B, self.Hq, self.Hkv, self.d, self.chunk, self.page,
            self.clusters, self.kmeans_iters, self.top_groups, self.top_pages, self.window,
            self.sinks, self.kv_bits, self.seed & (2**64 - 1), self.scale, self.head_shard, self.Tmax)

    @property
    def page_slots(self) -> int:
        return self.chunk // self.page + self.clusters

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv


class Index:
    """The sixteen device arrays of lod_index, as torch tensors (the arrays
    the parameters do not use are empty)."""

    def __init__(self, params: Params, device="cuda"):
        lib = load()
        sizes = (ctypes.c_size_t * len(_lib.INDEX_FIELDS))()
        check("lod_index_sizes", lib.lod_index_sizes(ctypes.byref(params.c()), sizes))
        p = params
        Cmax, k, P, d = p.Tmax // p.chunk, p.clusters, p.page_slots, p.d
        u = (p.B, p.Hkv)
        self.gK = torch.zeros(*u, Cmax * k, d, dtype=p.dtype, device=device)
        self.gV = torch.zeros_like(self.gK)
        self.gCnt = torch.zeros(*u, Cmax * k, dtype=torch.int32, device=device)
        self.pK = torch.zeros(*u, Cmax * P, d, dtype=p.dtype, device=device)
        self.pV = torch.zeros_like(self.pK)
        self.pCnt = torch.zeros(*u, Cmax * P, dtype=torch.int32, device=device)
        self.pBeg = torch.zeros(*u, Cmax * P, dtype=torch.int16, device=device)
        self.gPage = torch.zeros(*u, Cmax * (k + 1), dtype=torch.int16, device=device)
        self.perm = torch.full((*u, Cmax * p.chunk), -1, dtype=torch.int16, device=device)
        int4 = p.kv_bits == 4
        self.mK = torch.zeros(*u, 0 if int4 else Cmax * p.chunk, d, dtype=p.dtype, device=device)
        self.mV = torch.zeros_like(self.mK)
        self.gMeta = torch.zeros(*u, Cmax * k, dtype=torch.int32, device=device)
        self.qK = torch.zeros(*u, Cmax * p.chunk if int4 else 0, d // 2, dtype=torch.uint8, device=device)
        self.qV = torch.zeros_like(self.qK)
        self.qKs = torch.zeros(*u, Cmax * P if int4 else 0, d, 2, dtype=torch.float32, device=device)
        self.qVs = torch.zeros_like(self.qKs)
        for i, f in enumerate(_lib.INDEX_FIELDS):
            t = getattr(self, f)
            assert t.numel() * t.element_size() == sizes[i], (f, t.numel() * t.element_size(), sizes[i])

    def c(self) -> _lib.lod_index:
        return _lib.lod_index(*[getattr(self, f).data_ptr() for f in _lib.INDEX_FIELDS])

    def nbytes(self) -> int:
        return sum(getattr(self, f).numel() * getattr(self, f).element_size() for f in _lib.INDEX_FIELDS)


def workspace_bytes(params: Params, op: int) -> int:
    n = ctypes.c_size_t()
    check("lod_workspace_bytes", load().lod_workspace_bytes(ctypes.byref(params.c()), op, ctypes.byref(n)))
    return n.value


def workspace(params: Params, op: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace for `op` (LOD_OP_BUILD / _DECODE / _PREFILL)."""
    return torch.zeros(workspace_bytes(params, op), dtype=torch.uint8, device=device)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _kv_strides(params: Params, K: torch.Tensor, V: torch.Tensor):
    if K.dtype != params.dtype or V.dtype != params.dtype:
        raise TypeError("K/V dtype %s/%s != params dtype %s" % (K.dtype, V.dtype, params.dtype))
    if K.shape != V.shape or K.dim() != 4 or K.shape[:2] != (params.B, params.Hkv) or K.shape[3] != params.d:
        raise ValueError("K, V must be [B, Hkv, T, d]; got %s / %s" % (tuple(K.shape), tuple(V.shape)))
    if K.stride() != V.stride() or K.stride(3) != 1:
        raise ValueError("K and V must share strides with a contiguous last dimension")
    if K.shape[2] < params.Tmax:
        raise ValueError("KV cache holds %d tokens < Tmax %d" % (K.shape[2], params.Tmax))
    return (ctypes.c_int64 * 3)(K.stride(0), K.stride(1), K.stride(2))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def lod_build_index(params: Params, K, V, chunk_begin: int, chunk_end: int, index: Index, ws=None,
                    stream=None) -> None:
    """Build chunks [chunk_begin, chunk_end) of every (b, kvh) sequence."""
    lib = load()
    st = _kv_strides(params, K, V)
    if ws is None:
        ws = workspace(params, _lib.LOD_OP_BUILD, K.device)
    check("lod_build_index", lib.lod_build_index(
        ctypes.byref(params.c()), _ptr(K), _ptr(V), st, chunk_begin, chunk_end,
        ctypes.byref(index.c()), _ptr(ws), ws.numel(), _stream(stream)))


def lod_append_kv(params: Params, K, V, seq_lens, k_new, v_new, stream=None) -> None:
    """Write the current token's key/value rows k_new, v_new ([B, Hkv, d],
    cache dtype; on the device or in pinned host memory, which the kernel
    reads directly) into K/V at positions seq_lens - 1 (one kernel)."""
    lib = load()
    st = _kv_strides(params, K, V)
    shape = (params.B, params.Hkv, params.d)
    for t in (k_new, v_new):
        if t.shape != shape or t.dtype != params.dtype or not t.is_contiguous():
            raise ValueError("k_new / v_new must be contiguous %s %s" % (shape, params.dtype))
    check("lod_append_kv", lib.lod_append_kv(
        ctypes.byref(params.c()), _ptr(K), _ptr(V), st, _ptr(seq_lens), _ptr(k_new), _ptr(v_new),
        _stream(stream)))


def lod_build_ready(params: Params, K, V, seq_lens, index: Index, ws=None, stream=None) -> None:
    """Online build: for every sequence whose length (seq_lens, device int64
    [B]) is a positive multiple of the chunk, build the chunk it just
    completed; the decision is taken on the device, so this can be issued
    every decode step, e.g. on a second stream."""
    lib = load()
    st = _kv_strides(params, K, V)
    if seq_lens.shape != (params.B,) or seq_lens.dtype != torch.int64 or seq_lens.device != K.device:
        raise ValueError("seq_lens must be int64 [B] on the cache's device")
    if ws is None:
        ws = workspace(params, _lib.LOD_OP_BUILD, K.device)
    check("lod_build_ready", lib.lod_build_ready(
        ctypes.byref(params.c()), _ptr(K), _ptr(V), st, _ptr(seq_lens), ctypes.byref(index.c()),
        _ptr(ws), ws.numel(), _stream(stream)))


def lod_decode(params: Params, q, K, V, seq_lens, index: Index, out=None, lse=None, sel_groups=None,
               sel_pages=None, ws=None, stream=None):
    """One decode step: q [B, Hq, d] at positions seq_lens - 1.  Returns out.

    q and out may be pinned host tensors: the kernels then read q and store
    out over the host link themselves (no separate copy)."""
    lib = load()
    st = _kv_strides(params, K, V)
    if q.shape != (params.B, params.Hq, params.d) or q.dtype != params.dtype or not q.is_contiguous():
        raise ValueError("q must be contiguous [B, Hq, d] of the cache dtype")
    if seq_lens.dtype != torch.int64 or seq_lens.shape != (params.B,) or not seq_lens.is_cuda:
        raise ValueError("seq_lens must be a device int64 tensor [B]")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=K.device)
    if ws is None:
        ws = workspace(params, _lib.LOD_OP_DECODE, K.device)
    check("lod_decode", lib.lod_decode(
        ctypes.byref(params.c()), _ptr(q), _ptr(K), _ptr(V), st, _ptr(seq_lens),
        ctypes.byref(index.c()), _ptr(out), _ptr(lse), _ptr(sel_groups), _ptr(sel_pages), _ptr(ws),
        ws.numel(), _stream(stream)))
    return out


def lod_prefill(params: Params, q, q_begin: int, K, V, index: Index, out=None, lse=None,
                sel_groups=None, sel_pages=None, ws=None, stream=None):
    """Chunked causal prefill of q [B, Hq, Tq, d] at positions [q_begin, q_begin + Tq).
    Builds the index of the chunks completed in that range first.  Returns out."""
    lib = load()
    st = _kv_strides(params, K, V)
    if q.dim() != 4 or q.shape[:2] != (params.B, params.Hq) or q.shape[3] != params.d \
            or q.dtype != params.dtype or not q.is_contiguous():
        raise ValueError("q must be contiguous [B, Hq, Tq, d] of the cache dtype")
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, device=K.device)
    if ws is None:
        ws = workspace(params, _lib.LOD_OP_PREFILL, K.device)
    check("lod_prefill", lib.lod_prefill(
        ctypes.byref(params.c()), _ptr(q), q_begin, q.shape[2], _ptr(K), _ptr(V), st,
        ctypes.byref(index.c()), _ptr(out), _ptr(lse), _ptr(sel_groups), _ptr(sel_pages), _ptr(ws),
        ws.numel(), _stream(stream)))
    return out


def lod_get_status(ws, stream=None) -> int:
    """Read and clear the device status word (LOD_ST_* bits); synchronises."""
    v = ctypes.c_uint32()
    rc = load().lod_get_status(_ptr(ws), _stream(stream), ctypes.byref(v))
    if rc not in (_lib.LOD_OK, _lib.LOD_EDEVICE):
        check("lod_get_status", rc)
    return v.value
