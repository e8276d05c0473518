"""Parity at the full workload sizes, in the launch configuration the benchmark
times, on outputs the oracle can compute one by one.

  * GQA decode at 32K (batch 8) and at 128K (batch 4): the GPU builds the whole
    index and decodes the whole batch; sampled (sequence, KV head) units are
    rebuilt by the oracle (build compared under the k-means margin rule) and
    all their query heads are checked against the oracle on the GPU-built
    index (selections and outputs under the tie rule).
  * Chunked causal prefill of 131072 tokens: one lod_prefill call over the
    whole context; sampled rows (heads x positions, including chunk edges)
    are checked against the oracle.
  * Index build at 128K with k = 4 and k = 8: whole build, sampled KV heads
    compared chunk by chunk.
  * One sequence at a 1M-token context (inputs generated on the device).
"""
import numpy as np
import pytest
import torch

import oracle
from hierarchical_long_context_b200 import api, synth
from tests import lodtest as lt

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda")


def _np(t):
    return t.float().cpu().numpy()


@pytest.mark.parametrize("name, units, kv_bits", [
    ("decode_gqa_32k_bf16", [(0, 0), (5, 3), (7, 7)], 0),
    ("decode_gqa_128k_bf16", [(0, 1), (3, 6)], 0),
    ("decode_gqa_128k_bf16", [(1, 2), (2, 5)], 4),   # three-tier INT4
])
def test_decode_full_size(name, units, kv_bits):
    dev = _dev()
    w = synth.WORKLOADS[name]
    K, V = synth.kv_cache(w)
    p = lt.params_of(w, kv_bits=kv_bits)
    Kd, Vd = K.to(dev), V.to(dev)
    ix = api.Index(p, dev)
    api.lod_build_index(p, Kd, Vd, 0, w.T // 256, ix)
    q = synth.decode_queries(w).to(dev)
    sl = torch.full((w.B,), w.T, dtype=torch.int64, device=dev)
    lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
    sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
    sp = torch.empty(w.B, w.Hq, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE, dev)
    out = api.lod_decode(p, q, Kd, Vd, sl, ix, lse=lse, sel_groups=sg, sel_pages=sp, ws=ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    cfg = lt.oracle_cfg(w)
    nch = w.T // 256
    for b, h in units:
        Kn, Vn = _np(K[b, h]), _np(V[b, h])
        gu = lt.unit_from_gpu(ix, b, h, nch, p)
        ou = oracle.build_sequence(cfg, b * w.Hkv + h, Kn, Vn, nch)
        st = lt.compare_builds(gu, ou, cfg, True)
        assert st["diverged"] <= max(2, nch // 20), st
        if kv_bits == 4:
            lt.check_int4_pages(ix, b, h, gu, Kn, Vn, cfg)
            gu = lt.quantized(gu, Kn, Vn, cfg)
        rows = [(_np(q[b, hq]), w.T - 1, _np(out[b, hq]).astype(np.float64), float(lse[b, hq]),
                 sg[b, hq].cpu().numpy(), sp[b, hq].cpu().numpy()) for hq in range(h * w.g, (h + 1) * w.g)]
        print(name, (b, h), st, lt.check_rows(cfg, w.dtype, Kn, Vn, gu, rows))


def test_decode_1m_full_size():
    """One sequence at a 1M-token context (32760 visible groups per KV head):
    the GPU builds the whole index and decodes; one KV head is rebuilt by the
    oracle (build under the margin rule) and its 8 query heads checked."""
    dev = _dev()
    w = synth.WORKLOADS["decode_gqa_1m_bf16"]
    Kd, Vd = synth.kv_cache_device(w, dev)
    p = lt.params_of(w)
    ix = api.Index(p, dev)
    nch = w.T // 256
    api.lod_build_index(p, Kd, Vd, 0, nch, ix)
    q = synth.decode_queries(w).to(dev)
    sl = torch.full((w.B,), w.T, dtype=torch.int64, device=dev)
    lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
    sg = torch.empty(w.B, w.Hq, p.top_groups, dtype=torch.int32, device=dev)
    sp = torch.empty(w.B, w.Hq, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_DECODE, dev)
    out = api.lod_decode(p, q, Kd, Vd, sl, ix, lse=lse, sel_groups=sg, sel_pages=sp, ws=ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    cfg = lt.oracle_cfg(w)
    h = 5
    Kn, Vn = _np(Kd[0, h]), _np(Vd[0, h])
    gu = lt.unit_from_gpu(ix, 0, h, nch, p)
    ou = oracle.build_sequence(cfg, h, Kn, Vn, nch)
    st = lt.compare_builds(gu, ou, cfg, True)
    assert st["diverged"] <= max(2, nch // 20), st
    rows = [(_np(q[0, hq]), w.T - 1, _np(out[0, hq]).astype(np.float64), float(lse[0, hq]),
             sg[0, hq].cpu().numpy(), sp[0, hq].cpu().numpy()) for hq in range(h * w.g, (h + 1) * w.g)]
    print("1M", st, lt.check_rows(cfg, w.dtype, Kn, Vn, gu, rows))


def test_prefill_full_size():
    dev = _dev()
    w = synth.WORKLOADS["prefill_128k_bf16"]
    K, V = synth.kv_cache(w)
    p = lt.params_of(w)
    Kd, Vd = K.to(dev), V.to(dev)
    q = synth.prefill_queries(w, 0, w.T).to(dev)
    ix = api.Index(p, dev)
    lse = torch.empty(w.B, w.Hq, w.T, dtype=torch.float32, device=dev)
    sg = torch.empty(w.B, w.Hq, w.T, p.top_groups, dtype=torch.int32, device=dev)
    sp = torch.empty(w.B, w.Hq, w.T, p.top_groups, p.top_pages, dtype=torch.int32, device=dev)
    ws = api.workspace(p, api._lib.LOD_OP_PREFILL, dev)
    out = api.lod_prefill(p, q, 0, Kd, Vd, ix, lse=lse, sel_groups=sg, sel_pages=sp, ws=ws)
    torch.cuda.synchronize()
    assert api.lod_get_status(ws) == 0
    cfg = lt.oracle_cfg(w)
    nch = w.T // 256
    rng = np.random.default_rng(11)
    for h in (0, 5):
        Kn, Vn = _np(K[0, h]), _np(V[0, h])
        gu = lt.unit_from_gpu(ix, 0, h, nch, p)
        ts = sorted(set(rng.integers(0, w.T, 10).tolist()) | {255, 256, 767, 768, 65535, w.T - 1})
        rows = [(_np(q[0, hq, t]), t, _np(out[0, hq, t]).astype(np.float64), float(lse[0, hq, t]),
                 sg[0, hq, t].cpu().numpy(), sp[0, hq, t].cpu().numpy())
                for hq in (h * w.g, h * w.g + w.g - 1) for t in ts]
        print("prefill unit", h, lt.check_rows(cfg, w.dtype, Kn, Vn, gu, rows))


@pytest.mark.parametrize("k", [4, 8])
def test_build_full_size(k):
    dev = _dev()
    w = synth.WORKLOADS["build_128k_bf16"]
    K, V = synth.kv_cache(w)
    p = lt.params_of(w, k)
    Kd, Vd = K.to(dev), V.to(dev)
    ix = api.Index(p, dev)
    nch = w.T // 256
    api.lod_build_index(p, Kd, Vd, 0, nch, ix)
    torch.cuda.synchronize()
    cfg = lt.oracle_cfg(w, k)
    for h in (0, 7):
        Kn, Vn = _np(K[0, h]), _np(V[0, h])
        gu = lt.unit_from_gpu(ix, 0, h, nch, p)
        lt.check_index_consistency(gu, Kn, Vn, cfg, True)
        lt.check_member_copies(ix, 0, h, Kd[0, h], Vd[0, h], nch, p)
        ou = oracle.build_sequence(cfg, h, Kn, Vn, nch)
        st = lt.compare_builds(gu, ou, cfg, True)
        print("build k=%d kvh %d" % (k, h), st)
        assert st["keys_checked"] > 0.9 * nch * 200
        assert st["diverged"] <= max(2, nch // 20)
