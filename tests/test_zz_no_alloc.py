"""lod_decode_noalloc: decode for callers that cannot allocate device memory.

Engines that own every device allocation through their own pool, runtimes
that must not allocate while recording a CUDA graph or running a
latency-critical step, and plugin hosts that pass kernels only their inputs
and outputs cannot hand the library a workspace.  lod_decode_noalloc keeps
its scratch in an array built into the library instead.  These tests call it
through the C ABI and hold it to the workspace entry point's results.

This file is collected last on purpose (test_zz_...): if it fails, a run that
stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from hierarchical_long_context_b200 import _lib, api, synth
from tests import lodtest as lt


def _call(L, p, q, Kd, Vd, st, sl, ix, out, lse, sg, sp, status=None):
    return L.lod_decode_noalloc(
        ctypes.byref(p.c()), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(Kd.data_ptr()),
        ctypes.c_void_p(Vd.data_ptr()), st, ctypes.c_void_p(sl.data_ptr()), ctypes.byref(ix.c()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(sg.data_ptr()),
        ctypes.c_void_p(sp.data_ptr()),
        ctypes.c_void_p(status.data_ptr()) if status is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_a_misaligned_status_word_is_rejected_without_touching_a_gpu():
    """The kernels OR status bits into the caller's word with 4-byte atomics:
    a pointer off a 4-byte boundary is refused before anything is enqueued."""
    L = _lib.load()
    p = api.Params(B=1, Hq=8, Hkv=1, d=128, Tmax=4096)
    assert api.workspace_bytes(p, _lib.LOD_OP_DECODE) <= _lib.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    full = _lib.lod_index(*([1 << 20] * len(_lib.INDEX_FIELDS)))
    st = (ctypes.c_int64 * 3)(4096 * 128, 4096 * 128, 128)  # fake, never used
    rc = L.lod_decode_noalloc(ctypes.byref(p.c()), fake, fake, fake, st, fake, ctypes.byref(full), fake,
                              None, None, None, ctypes.c_void_p((1 << 20) + 2), None)
    assert rc == _lib.LOD_EINVAL
    assert "status" in L.lod_last_error().decode()


def test_shapes_beyond_the_built_in_scratch_are_rejected_without_touching_a_gpu():
    L = _lib.load()
    # 512 sequences x 8 KV heads need more split states than the built-in array holds
    p = api.Params(B=512, Hq=64, Hkv=8, d=128, Tmax=1 << 20)
    assert api.workspace_bytes(p, _lib.LOD_OP_DECODE) > _lib.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    full = _lib.lod_index(*([1 << 20] * len(_lib.INDEX_FIELDS)))
    st = (ctypes.c_int64 * 3)(8 * (1 << 20) * 128, (1 << 20) * 128, 128)  # fake, never used
    rc = L.lod_decode_noalloc(ctypes.byref(p.c()), fake, fake, fake, st, fake, ctypes.byref(full), fake,
                              None, None, None, None, None)
    assert rc == _lib.LOD_EINVAL
    msg = L.lod_last_error().decode()
    assert "exceeds" in msg and str(_lib.NOALLOC_SCRATCH_BYTES) in msg


@pytest.mark.gpu
def test_noalloc_decode_matches_the_workspace_decode_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda")
    L = _lib.load()
    w = synth.WORKLOADS["decode_gqa_32k_bf16"].with_(B=2, Hkv=2, Hq=16)
    T = 8192
    Kc, Vc = synth.kv_cache(w, T)
    p = lt.params_of(w, Tmax=T)
    assert api.workspace_bytes(p, _lib.LOD_OP_DECODE) <= _lib.NOALLOC_SCRATCH_BYTES
    Kd, Vd = Kc.to(dev), Vc.to(dev)
    ix = api.Index(p)
    api.lod_build_index(p, Kd, Vd, 0, T // 256, ix)
    st = (ctypes.c_int64 * 3)(Kd.stride(0), Kd.stride(1), Kd.stride(2))
    sl = torch.tensor([T, T - 777], dtype=torch.int64, device=dev)
    tol = lt.TOL[w.dtype]
    for call in range(2):
        q = synth.decode_queries(w, stream="noalloc%d" % call).to(dev)
        # reference: the workspace entry point
        ref_lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
        ref_sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
        ref_sp = torch.empty(w.B, w.Hq, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
        ref = api.lod_decode(p, q, Kd, Vd, sl, ix, lse=ref_lse, sel_groups=ref_sg, sel_pages=ref_sp)
        # the entry point under test, straight through the C ABI
        out = torch.full_like(q, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        sg = torch.full_like(ref_sg, -7)
        sp = torch.full_like(ref_sp, -7)
        status = torch.zeros(1, dtype=torch.int32, device=dev) if call == 0 else None
        rc = _call(L, p, q, Kd, Vd, st, sl, ix, out, lse, sg, sp, status)
        assert rc == _lib.LOD_OK, L.lod_last_error()
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the results are bit-identical
        # (a scratch-layout error smaller than the parity tolerance would
        # still show here); the tolerance only sizes the failure message
        err = (out.float() - ref.float()).abs().max().item()
        assert torch.equal(out, ref), "call %d: max-abs %.3g (tolerance %g)" % (call, err, tol)
        assert torch.isfinite(out.float()).all()
        assert torch.equal(lse, ref_lse), np.max(np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()))
        assert torch.equal(sg, ref_sg) and torch.equal(sp, ref_sp)
        if status is not None:
            assert int(status.item()) == 0
